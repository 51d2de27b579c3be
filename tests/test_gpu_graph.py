"""Decode steps captured once in a CUDA graph and replayed with new inputs.

A serving loop (and the benchmark) captures a step, the per-token K/V append
followed by the attention call, through the public API and replays it: the plan
kernel, the attention kernel and the merge are programmatic dependent launches
inside the graph, and every replay reads that step's lengths, slots, new rows and
queries from the same device buffers.  Each replay's output is compared with the
oracle run on the host-side state (the host pools advanced by the oracle's own
append), so that a plan, workspace or launch-order problem of the replayed graph
shows up as a wrong result.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_328_b200 as pkv
from paged_kv_cache_328_b200 import workloads as wl
from paritykit import TOL

pytestmark = pytest.mark.gpu

STEPS = 4


@pytest.fixture(scope="module")
def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pkv.load()
    return torch.device("cuda", 0)


# (K/V heads, query heads, dtype, partition tokens): multi-head on the CUDA-core kernel (split
# and unsplit), G = 4 on the warp-level kernel, G = 8 and 32 on the token-major kernel
CASES = [(4, 4, "f16", 0), (4, 4, "f16", 64), (2, 8, "bf16", 0), (2, 16, "bf16", 128), (2, 64, "bf16", 0)]


@pytest.mark.parametrize("Hkv,Hq,dtype,pt", CASES)
def test_replayed_step_graph(dev, Hkv, Hq, dtype, pt):
    S, D, B = 40, 128, 16
    rng = np.random.default_rng(4100 + Hq + pt)
    c0 = rng.integers(0, 400, S)
    c0[:3] = [0, 15, 16]  # empty, one short of a block, a full block: the next token opens / fills one
    final = c0 + STEPS
    # tables and pool for the final lengths; each step writes its token's rows over that position
    w = wl.build_paged(final, H=Hkv, D=D, B=B, dtype=dtype, seed=4200 + Hq, device=dev, num_q_heads=Hq)
    bt = torch.from_numpy(w.block_tables).to(dev)
    tdt = w.q.dtype
    # static buffers the graph reads
    q_buf = torch.zeros((S, Hq, D), dtype=tdt, device=dev)
    k_buf = torch.zeros((S, Hkv, D), dtype=tdt, device=dev)
    v_buf = torch.zeros((S, Hkv, D), dtype=tdt, device=dev)
    slot_buf = torch.full((S,), -1, dtype=torch.int64, device=dev)
    ctx_buf = torch.zeros((S,), dtype=torch.int32, device=dev)
    out = torch.zeros((S, Hq, D), dtype=torch.float32, device=dev)
    ws = pkv.alloc_workspace(q_buf, w.k_pool, bt, pt)

    def step():
        pkv.kv_cache_append(k_buf, v_buf, w.k_pool, w.v_pool, slot_buf)
        pkv.paged_attn_decode(q_buf, w.k_pool, w.v_pool, bt, ctx_buf, w.scale, out=out, partition_tokens=pt,
                              workspace=ws)

    host_k, host_v = w.host(w.k_pool), w.host(w.v_pool)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step()  # warm-up outside the capture (all slots -1, every context empty)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            step()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    try:
        for t in range(STEPS):
            ctx = (c0 + t + 1).astype(np.int64)
            pos = ctx - 1
            slots = w.block_tables[np.arange(S), pos // B].astype(np.int64) * B + pos % B
            gen = torch.Generator().manual_seed(4300 + 10 * t + Hq)
            q_t = torch.randn((S, Hq, D), generator=gen).to(tdt)
            k_t = torch.randn((S, Hkv, D), generator=gen).to(tdt)
            v_t = torch.randn((S, Hkv, D), generator=gen).to(tdt)
            q_buf.copy_(q_t)
            k_buf.copy_(k_t)
            v_buf.copy_(v_t)
            slot_buf.copy_(torch.from_numpy(slots))
            ctx_buf.copy_(torch.from_numpy(ctx.astype(np.int32)))
            out.fill_(float("nan"))
            g.replay()
            torch.cuda.synchronize()
            code, reason = pkv.get_device_error(dev)
            assert code == 0, (t, code, reason)
            host_k, host_v, n_bad = oracle.kv_append(host_k, host_v, w.host(k_t), w.host(v_t), slots, B)
            assert n_bad == 0
            want = oracle.paged_decode(w.host(q_t), host_k, host_v, w.block_tables, ctx, w.scale, B, dtype)
            got = out.cpu().numpy()
            assert np.all(np.isfinite(got)), t
            err = float(np.max(np.abs(got - want)))
            assert err <= TOL[dtype], (t, err)
    finally:
        del g
