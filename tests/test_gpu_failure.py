"""GPU: a stalled pipeline wait ends with an error status, not a hang.

Every mbarrier wait in the attention kernels is bounded; when one runs out the
kernel records PKV_DEV_WAIT_TIMEOUT in the device error word and returns.  The
self-test kernel waits on a barrier that nothing arrives on (no fault, no trap),
and the test checks the status, that reading it clears it, and that the context
still runs a decode correctly afterwards.
"""

import time

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_328_b200 as pkv
from paged_kv_cache_328_b200 import workloads as wl
from paritykit import TOL, dev_indices, max_err

pytestmark = pytest.mark.gpu

PKV_ETIMEOUT = -8
PKV_DEV_WAIT_TIMEOUT = 5


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pkv.load()
    return torch.device("cuda", 0)


def test_stalled_wait_times_out_and_context_survives(dev):
    assert pkv.get_device_error(dev) == (0, 0)
    t0 = time.perf_counter()
    assert pkv.selftest_wait_timeout(20_000_000, device=dev)   # ~10 ms at 2 GHz
    took = time.perf_counter() - t0
    assert took < 5.0, took
    assert pkv.get_device_error(dev) == (PKV_ETIMEOUT, PKV_DEV_WAIT_TIMEOUT)
    assert pkv.get_device_error(dev) == (0, 0)                  # reading cleared it

    w = wl.build_paged([5, 300, 0, 77], 4, 128, 16, "bf16", 3, device=dev)
    ix = dev_indices(w, dev)
    got = pkv.paged_attn_decode(w.q, w.k_pool, w.v_pool, ix["bt"], ix["ctx"], w.scale).cpu().numpy()
    want = oracle.paged_decode(w.host(w.q), w.host(w.k_pool), w.host(w.v_pool), w.block_tables, w.context_lens,
                               w.scale, w.B, w.dtype)
    assert max_err(got, want) <= TOL["bf16"]
    assert pkv.get_device_error(dev) == (0, 0)


def test_longer_limit_waits_longer(dev):
    t = []
    for limit in (2_000_000, 200_000_000):                        # ~1 ms, ~100 ms
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        assert pkv.selftest_wait_timeout(limit, device=dev)
        t.append(time.perf_counter() - t0)
        assert pkv.get_device_error(dev) == (PKV_ETIMEOUT, PKV_DEV_WAIT_TIMEOUT)
    assert t[1] > t[0] and t[1] > 0.02, t
