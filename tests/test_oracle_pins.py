"""Pins for the CPU oracle against what the pages and the mathematics fix.

None of these checks re-uses the oracle's own code path to produce an expected
value.  The expected values come from:

* the pages' worked block tables, written out by hand in ``tests/golden/``;
* the IEEE 754 / bfloat16 bit-field definitions (storage widening);
* brute force in pure Python over a flat memory buffer with ``math.fsum``;
* a library routine (``torch.nn.functional.scaled_dot_product_attention`` in
  float64) on contiguous data placed into the pool by test code;
* closed forms: one-token context, q = 0, two tokens (logistic weight), a
  dominant key, the empty context;
* invariants: any physical permutation and any block size give bit-identical
  results, because paging only changes where tokens live ("PagedAttention -
  Efficient Memory Management for LLM Serving with vLLM", framework-overview
  flowchart: logical blocks are contiguous for the sequence, physical blocks
  sit anywhere).

``test_planted_mistakes_are_caught`` plants plausible mistakes in the oracle
(on the CPU, by monkeypatching) and checks that at least one pin fails for each.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import cache_ops, paged_attention, storage

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------------------
# Test-side helpers (independent of the oracle)
# ---------------------------------------------------------------------------

def load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def encoded_pool(nb, H, B, D):
    """Pool element (p, h, o, d) = 10000*h + 100*p + o + d/8 (exact in float32)."""
    p = np.arange(nb)[:, None, None, None]
    h = np.arange(H)[None, :, None, None]
    o = np.arange(B)[None, None, :, None]
    d = np.arange(D)[None, None, None, :]
    return (10000.0 * h + 100.0 * p + o + d / 8.0).astype(np.float32)


def location_of(row, h):
    """(block, slot) named by a row of an encoded pool."""
    base = float(row[0]) - 10000.0 * h
    p = int(base // 100)
    o = int(round(base - 100 * p))
    return p, o


def expand_ranges(ranges):
    out = []
    for r in ranges:
        t0, t1 = r["logical_tokens"]
        for i, t in enumerate(range(t0, t1 + 1)):
            out.append((t, r["physical_block"], r["first_slot"] + i))
    return out


def random_stored(rng, shape, dtype):
    """Random finite stored elements: float32, or uint16 bit patterns of fp16 / bf16."""
    x = rng.standard_normal(shape).astype(np.float32)
    if dtype == "f32":
        return x
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    return (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def place_flat(K, V, B, nb, table, dtype):
    """Scatter contiguous per-head rows ``[H, ctx, D]`` into NaN-filled pools.

    Written with explicit flat offsets ((phys*H + h)*B + t%B)*D so that it does
    not share the oracle's indexing.
    """
    H, ctx, D = K.shape
    fill = np.float32(np.nan) if dtype == "f32" else np.uint16(0x7FC0 if dtype == "bf16" else 0x7E00)
    kf = np.full(nb * H * B * D, fill, dtype=K.dtype)
    vf = np.full(nb * H * B * D, fill, dtype=V.dtype)
    for t in range(ctx):
        phys = table[t // B]
        for h in range(H):
            start = ((phys * H + h) * B + t % B) * D
            kf[start:start + D] = K[h, t]
            vf[start:start + D] = V[h, t]
    return kf.reshape(nb, H, B, D), vf.reshape(nb, H, B, D)


def random_table(rng, nb, nblocks):
    return [int(x) for x in rng.permutation(nb)[:nblocks]]


def ieee_half(bits):
    """binary16 value from its sign/exponent/mantissa fields (IEEE 754 definition)."""
    s = (bits >> 15) & 1
    e = (bits >> 10) & 0x1F
    m = bits & 0x3FF
    if e == 0:
        v = math.ldexp(m / 1024.0, -14)
    else:
        v = math.ldexp(1.0 + m / 1024.0, e - 15)
    return -v if s else v


def bfloat16_value(bits):
    """bfloat16 value from its fields: 1 sign, 8 exponent (bias 127), 7 mantissa bits."""
    s = (bits >> 15) & 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    if e == 0:
        v = math.ldexp(m / 128.0, -126)
    else:
        v = math.ldexp(1.0 + m / 128.0, e - 127)
    return -v if s else v


# ---------------------------------------------------------------------------
# Pin checks (plain functions so the planted-mistake test can re-run them)
# ---------------------------------------------------------------------------

def check_storage_f16():
    bits = np.array([b for b in range(1 << 16) if ((b >> 10) & 0x1F) != 0x1F], dtype=np.uint16)
    got = storage.to_f64(bits, "f16")
    want = np.array([ieee_half(int(b)) for b in bits])
    assert np.array_equal(got, want)


def check_storage_bf16():
    bits = np.array([b for b in range(1 << 16) if ((b >> 7) & 0xFF) != 0xFF], dtype=np.uint16)
    got = storage.to_f64(bits, "bf16")
    want = np.array([bfloat16_value(int(b)) for b in bits])
    assert np.array_equal(got, want)
    # a library routine agrees too
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got, lib)


def check_golden_velog(golden_dir):
    g = load(golden_dir, "velog_block_table.json")
    pool = encoded_pool(g["num_blocks"], g["num_heads"], g["block_size"], g["head_dim"])
    want = expand_ranges(g["expected"])
    assert len(want) == g["context_len"]
    for h in range(g["num_heads"]):
        rows = oracle.gather_rows(pool, g["table"], g["context_len"], h, g["block_size"])
        assert rows.shape == (g["context_len"], g["head_dim"])
        for t, blk, slot in want:
            assert location_of(rows[t], h) == (blk, slot), (h, t)
            assert np.array_equal(rows[t], pool[blk, h, slot])


def check_golden_digest(golden_dir):
    g = load(golden_dir, "digest_flowchart.json")
    nb, H, B, D = g["num_blocks"], g["num_heads"], g["block_size"], g["head_dim"]
    kpool = encoded_pool(nb, H, B, D)
    vpool = kpool + np.float32(0.5)
    for seq, table in g["tables"].items():
        ctx = g["context_lens"][seq]
        want = expand_ranges(g["expected_gather"][seq])
        got = oracle.gather_kv(kpool, table, ctx, B)
        for h in range(H):
            for t, blk, slot in want:
                assert location_of(got[h, t], h) == (blk, slot)
    # copy-on-write P3 -> P9: the copy equals the source, nothing else changes
    src, dst = g["cow_pair"]
    k2, v2, bad = oracle.kv_block_copy(kpool, vpool, np.array([[src, dst]]))
    assert bad == 0
    assert np.array_equal(k2[dst], kpool[src]) and np.array_equal(v2[dst], vpool[src])
    for b in range(nb):
        if b != dst:
            assert np.array_equal(k2[b], kpool[b]) and np.array_equal(v2[b], vpool[b])
    # sequence 2 pointed at its copy reads the same tokens as before
    before = oracle.gather_kv(vpool, g["tables"]["seq2"], g["context_lens"]["seq2"], B)
    after = oracle.gather_kv(v2, g["table_after_cow"]["seq2"], g["context_lens"]["seq2"], B)
    assert np.array_equal(before, after)
    # appends land where the table says and extend the logical sequence by one token
    for a in g["append"]:
        seq = a["seq"]
        table = g["tables"][seq]
        ctx = g["context_lens"][seq]
        newk = np.full((1, H, D), -7.0, dtype=np.float32)
        newv = np.full((1, H, D), -9.0, dtype=np.float32)
        k3, v3, bad = oracle.kv_append(kpool, vpool, newk, newv, np.array([a["slot"]]), B)
        assert bad == 0
        rows = oracle.gather_kv(v3, table, ctx + 1, B)
        assert np.all(rows[:, ctx] == -9.0)
        assert np.array_equal(rows[:, :ctx], oracle.gather_kv(vpool, table, ctx, B))
        changed = np.argwhere(np.any(k3 != kpool, axis=-1))
        assert changed.tolist() == [[a["slot"] // B, h, a["slot"] % B] for h in range(H)]


def check_golden_on_demand(golden_dir):
    g = load(golden_dir, "velog_on_demand.json")
    nb, H, B, D = g["num_blocks"], g["num_heads"], g["block_size"], g["head_dim"]
    k = np.full((nb, H, B, D), np.nan, dtype=np.float32)
    v = np.full((nb, H, B, D), np.nan, dtype=np.float32)
    for t, slot in enumerate(g["expected_slots"]):
        kn = np.full((1, H, D), t, dtype=np.float32)
        vn = np.full((1, H, D), 100 + t, dtype=np.float32)
        k, v, bad = oracle.kv_append(k, v, kn, vn, np.array([slot]), B)
        assert bad == 0
    rows_k = oracle.gather_kv(k, g["expected_table"], g["tokens"], B)
    rows_v = oracle.gather_kv(v, g["expected_table"], g["tokens"], B)
    for t in range(g["tokens"]):
        assert np.all(rows_k[:, t] == t) and np.all(rows_v[:, t] == 100 + t)
    # only the slots written hold data; the last block is the only partial one
    assert int(np.sum(~np.isnan(k[:, 0, :, 0]))) == g["tokens"]


def brute_force_decode(kflat, vflat, qflat, tables, ctxs, H, D, B, scale, to64):
    """Pure-Python paged attention over flat buffers, summed with math.fsum."""
    S = len(ctxs)
    out = np.zeros((S, H, D))
    for s in range(S):
        for h in range(H):
            ctx = ctxs[s]
            if ctx == 0:
                continue
            qv = [to64(qflat[(s * H + h) * D + d]) for d in range(D)]
            logits = []
            rows = []
            for t in range(ctx):
                phys = tables[s][t // B]
                base = ((phys * H + h) * B + t % B) * D
                krow = [to64(kflat[base + d]) for d in range(D)]
                rows.append([to64(vflat[base + d]) for d in range(D)])
                logits.append(scale * math.fsum(qv[d] * krow[d] for d in range(D)))
            m = max(logits)
            e = [math.exp(x - m) for x in logits]
            z = math.fsum(e)
            for d in range(D):
                out[s, h, d] = math.fsum(e[t] * rows[t][d] for t in range(ctx)) / z
    return out


def check_brute_force_tiny():
    """Config-1 shapes: 4 sequences, 2 heads x 64, fp32, B=16, 16-block pool."""
    rng = np.random.default_rng(11)
    H, D, B, nb = 2, 64, 16, 16
    ctxs = [1, 15, 16, 37]
    perm = rng.permutation(nb)
    tables, cur = [], 0
    for c in ctxs:
        n = -(-c // B)
        tables.append([int(x) for x in perm[cur:cur + n]] + [-1] * (3 - n))
        cur += n
    kflat = rng.standard_normal(nb * H * B * D).astype(np.float32)
    vflat = rng.standard_normal(nb * H * B * D).astype(np.float32)
    qflat = rng.standard_normal(len(ctxs) * H * D).astype(np.float32)
    want = brute_force_decode(kflat, vflat, qflat, tables, ctxs, H, D, B, 1.0 / 8.0, float)
    got = oracle.paged_decode(qflat.reshape(len(ctxs), H, D), kflat.reshape(nb, H, B, D),
                              vflat.reshape(nb, H, B, D), np.array(tables), np.array(ctxs),
                              1.0 / 8.0, B, "f32")
    assert np.max(np.abs(got - want)) <= 1e-12


def check_sdpa_library(dtype):
    """Paged oracle == library attention on the contiguous rows that test code placed."""
    rng = np.random.default_rng(12)
    H, D, B, nb = 3, 64, 16, 24
    for ctx in (1, 2, 15, 16, 17, 33, 100):
        K = random_stored(rng, (H, ctx, D), dtype)
        V = random_stored(rng, (H, ctx, D), dtype)
        q = random_stored(rng, (1, H, D), dtype)
        table = random_table(rng, nb, -(-ctx // B))
        kp, vp = place_flat(K, V, B, nb, table, dtype)
        scale = 1.0 / math.sqrt(D)
        got = oracle.paged_decode(q, kp, vp, np.array([table]), np.array([ctx]), scale, B, dtype)[0]
        qt = torch.from_numpy(storage_lib(q[0], dtype))[:, None, :]
        Kt = torch.from_numpy(storage_lib(K, dtype))
        Vt = torch.from_numpy(storage_lib(V, dtype))
        ref = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)[:, 0, :]
        assert np.max(np.abs(got - ref.numpy())) <= 1e-12, ctx


def storage_lib(x, dtype):
    """Stored elements -> float64 through torch's own dtype conversion (a library routine)."""
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float64).numpy()
    tdt = torch.float16 if dtype == "f16" else torch.bfloat16
    return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(tdt).to(torch.float64).numpy()


def _one_seq(rng, ctx, H=2, D=64, B=16, nb=12, dtype="f32", q=None, K=None, V=None):
    K = random_stored(rng, (H, ctx, D), dtype) if K is None else K
    V = random_stored(rng, (H, ctx, D), dtype) if V is None else V
    q = random_stored(rng, (1, H, D), dtype) if q is None else q
    table = random_table(rng, nb, max(1, -(-ctx // B)))
    kp, vp = place_flat(K, V, B, nb, table, dtype)
    return q, K, V, kp, vp, table


def check_one_token_returns_v():
    rng = np.random.default_rng(13)
    for dtype in ("f32", "f16", "bf16"):
        q, K, V, kp, vp, table = _one_seq(rng, 1, dtype=dtype)
        got = oracle.paged_decode(q, kp, vp, np.array([table]), np.array([1]), 0.125, 16, dtype)[0]
        assert np.array_equal(got, storage_lib(V[:, 0, :], dtype))


def check_zero_query_gives_mean():
    rng = np.random.default_rng(14)
    for ctx in (3, 16, 29):
        q0 = np.zeros((1, 2, 64), dtype=np.float32)
        q, K, V, kp, vp, table = _one_seq(rng, ctx, q=q0)
        got = oracle.paged_decode(q, kp, vp, np.array([table]), np.array([ctx]), 0.125, 16, "f32")[0]
        for h in range(2):
            for d in range(64):
                mean = math.fsum(float(V[h, t, d]) for t in range(ctx)) / ctx
                assert abs(got[h, d] - mean) <= 1e-12


def check_two_tokens_logistic():
    rng = np.random.default_rng(15)
    q, K, V, kp, vp, table = _one_seq(rng, 2)
    scale = 0.125
    got = oracle.paged_decode(q, kp, vp, np.array([table]), np.array([2]), scale, 16, "f32")[0]
    for h in range(2):
        x0 = scale * math.fsum(float(q[0, h, d]) * float(K[h, 0, d]) for d in range(64))
        x1 = scale * math.fsum(float(q[0, h, d]) * float(K[h, 1, d]) for d in range(64))
        sig = 1.0 / (1.0 + math.exp(-(x1 - x0)))   # weight of token 1
        for d in range(64):
            v0, v1 = float(V[h, 0, d]), float(V[h, 1, d])
            assert abs(got[h, d] - (v0 + sig * (v1 - v0))) <= 1e-12


def check_dominant_key():
    """One key aligned with q and a large scale: |out - V_j| <= (n-1) e^{-gap} max|V_i - V_j|."""
    rng = np.random.default_rng(16)
    ctx, D = 20, 64
    K = rng.standard_normal((1, ctx, D)).astype(np.float32) * np.float32(0.01)
    j = 13
    K[0, j] = np.float32(1.0)
    q = np.ones((1, 1, D), dtype=np.float32)
    V = rng.standard_normal((1, ctx, D)).astype(np.float32)
    q, K, V, kp, vp, table = _one_seq(rng, ctx, H=1, q=q, K=K, V=V)
    scale = 0.5
    got = oracle.paged_decode(q, kp, vp, np.array([table]), np.array([ctx]), scale, 16, "f32")[0, 0]
    x = [scale * math.fsum(float(K[0, t, d]) for d in range(D)) for t in range(ctx)]
    gap = x[j] - max(x[t] for t in range(ctx) if t != j)
    bound = (ctx - 1) * math.exp(-gap) * float(np.max(np.abs(V[0] - V[0, j])))
    assert gap > 20
    assert np.max(np.abs(got - V[0, j].astype(np.float64))) <= bound + 1e-15
    assert not np.array_equal(got, V[0, j].astype(np.float64)) or bound < 1e-300


def check_empty_context_zero():
    nb, H, B, D = 4, 2, 16, 8
    pool = np.full((nb, H, B, D), np.nan, dtype=np.float32)
    q = np.ones((1, H, D), dtype=np.float32)
    got = oracle.paged_decode(q, pool, pool, np.array([[-1]]), np.array([0]), 1.0, B, "f32")
    assert np.array_equal(got, np.zeros((1, H, D)))


def check_permutation_invariance():
    rng = np.random.default_rng(17)
    for dtype in ("f32", "f16", "bf16"):
        ctx, H, D, B, nb = 45, 2, 64, 16, 10
        K = random_stored(rng, (H, ctx, D), dtype)
        V = random_stored(rng, (H, ctx, D), dtype)
        q = random_stored(rng, (1, H, D), dtype)
        outs = []
        for _ in range(4):
            table = random_table(rng, nb, 3)
            kp, vp = place_flat(K, V, B, nb, table, dtype)
            outs.append(oracle.paged_decode(q, kp, vp, np.array([table]), np.array([ctx]),
                                            0.125, B, dtype))
        for o in outs[1:]:
            assert np.array_equal(o, outs[0])


def check_block_size_invariance():
    rng = np.random.default_rng(18)
    ctx, H, D = 150, 2, 64
    for dtype in ("f16", "bf16"):
        K = random_stored(rng, (H, ctx, D), dtype)
        V = random_stored(rng, (H, ctx, D), dtype)
        q = random_stored(rng, (1, H, D), dtype)
        outs = []
        for B in (8, 16, 32, 64, 128):
            nblk = -(-ctx // B)
            nb = nblk + 3
            table = random_table(rng, nb, nblk)
            kp, vp = place_flat(K, V, B, nb, table, dtype)
            outs.append(oracle.paged_decode(q, kp, vp, np.array([table]), np.array([ctx]),
                                            0.125, B, dtype))
        for o in outs[1:]:
            assert np.array_equal(o, outs[0])


def check_append_brute_force():
    rng = np.random.default_rng(19)
    nb, H, B, D, T = 6, 3, 8, 16, 10
    k = rng.standard_normal((nb, H, B, D)).astype(np.float32)
    v = rng.standard_normal((nb, H, B, D)).astype(np.float32)
    kn = rng.standard_normal((T, H, D)).astype(np.float32)
    vn = rng.standard_normal((T, H, D)).astype(np.float32)
    slots = rng.choice(nb * B, size=T, replace=False).astype(np.int64)
    slots[3] = -1
    slots[7] = nb * B + 5            # out of range: skipped and counted
    k2, v2, bad = oracle.kv_append(k, v, kn, vn, slots, B)
    assert bad == 1
    kf, vf = k.reshape(-1).copy(), v.reshape(-1).copy()
    for t in range(T):
        s = int(slots[t])
        if s < 0 or s >= nb * B:
            continue
        blk, off = s // B, s % B
        for h in range(H):
            start = ((blk * H + h) * B + off) * D
            kf[start:start + D] = kn[t, h]
            vf[start:start + D] = vn[t, h]
    assert np.array_equal(k2.reshape(-1), kf) and np.array_equal(v2.reshape(-1), vf)


def check_block_copy_brute_force():
    rng = np.random.default_rng(20)
    nb, H, B, D = 9, 2, 4, 8
    k = rng.standard_normal((nb, H, B, D)).astype(np.float32)
    v = rng.standard_normal((nb, H, B, D)).astype(np.float32)
    pairs = np.array([[1, 5], [2, 7], [0, 3], [4, nb]])   # the last pair is out of range
    k2, v2, bad = oracle.kv_block_copy(k, v, pairs)
    assert bad == 1
    size = H * B * D
    kf, vf = k.reshape(-1).copy(), v.reshape(-1).copy()
    for src, dst in pairs[:3]:
        kf[dst * size:(dst + 1) * size] = k.reshape(-1)[src * size:(src + 1) * size]
        vf[dst * size:(dst + 1) * size] = v.reshape(-1)[src * size:(src + 1) * size]
    assert np.array_equal(k2.reshape(-1), kf) and np.array_equal(v2.reshape(-1), vf)


def check_gqa_equals_replicated_mha():
    """Grouped-query attention is multi-head attention with each K/V head repeated G times."""
    rng = np.random.default_rng(22)
    Hq, Hkv, D, B, nb, ctx = 8, 2, 64, 16, 12, 70
    G = Hq // Hkv
    for dtype in ("f16", "bf16"):
        K = random_stored(rng, (Hkv, ctx, D), dtype)
        V = random_stored(rng, (Hkv, ctx, D), dtype)
        q = random_stored(rng, (1, Hq, D), dtype)
        table = random_table(rng, nb, -(-ctx // B))
        kp, vp = place_flat(K, V, B, nb, table, dtype)
        kr, vr = place_flat(np.repeat(K, G, axis=0), np.repeat(V, G, axis=0), B, nb, table, dtype)
        gqa = oracle.paged_decode(q, kp, vp, np.array([table]), np.array([ctx]), 0.125, B, dtype)
        mha = oracle.paged_decode(q, kr, vr, np.array([table]), np.array([ctx]), 0.125, B, dtype)
        assert np.array_equal(gqa, mha)
        # and against the library routine, grouped the same way
        qt = torch.from_numpy(storage_lib(q[0], dtype))[:, None, :]
        Kt = torch.from_numpy(storage_lib(K, dtype)).repeat_interleave(G, dim=0)
        Vt = torch.from_numpy(storage_lib(V, dtype)).repeat_interleave(G, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=0.125)[:, 0, :]
        assert np.max(np.abs(gqa[0] - ref.numpy())) <= 1e-12


def check_multi_query_rows_are_shorter_decodes():
    """Query token j of Lq sees the first ctx - Lq + j + 1 tokens: each row equals the
    decode oracle over that shorter context, and the last row equals decode over ctx."""
    rng = np.random.default_rng(23)
    Hq, Hkv, D, B, nb = 4, 2, 64, 16, 14
    for dtype in ("f16", "bf16"):
        ctxs = [7, 40, 3]
        Lq = 5
        tables = []
        perm = rng.permutation(nb)
        cur = 0
        for c in ctxs:
            n = -(-c // B)
            tables.append([int(x) for x in perm[cur:cur + n]] + [-1] * (3 - n))
            cur += n
        kp = random_stored(rng, (nb, Hkv, B, D), dtype)
        vp = random_stored(rng, (nb, Hkv, B, D), dtype)
        q = random_stored(rng, (len(ctxs), Lq, Hq, D), dtype)
        got = oracle.paged_multi_query(q, kp, vp, np.array(tables), np.array(ctxs), 0.125, B, dtype)
        for s, c in enumerate(ctxs):
            for j in range(Lq):
                vis = max(0, c - Lq + j + 1)
                dec = oracle.paged_decode(q[s:s + 1, j], kp, vp, np.array([tables[s]]), np.array([vis]),
                                          0.125, B, dtype)[0]
                assert np.array_equal(got[s, j], dec), (s, j)
        # brute force for one row of a sequence whose context is longer than Lq
        s, j, h = 1, 2, 3
        vis = ctxs[s] - Lq + j + 1
        qv = storage_lib(q[s, j, h], dtype)
        logits, rows = [], []
        for t in range(vis):
            blk, off = tables[s][t // B], t % B
            kr = storage_lib(kp[blk, h // (Hq // Hkv), off], dtype)
            rows.append(storage_lib(vp[blk, h // (Hq // Hkv), off], dtype))
            logits.append(0.125 * math.fsum(float(qv[d]) * float(kr[d]) for d in range(D)))
        m = max(logits)
        e = [math.exp(x - m) for x in logits]
        z = math.fsum(e)
        want = [math.fsum(e[t] * float(rows[t][d]) for t in range(vis)) / z for d in range(D)]
        assert np.max(np.abs(got[s, j, h] - np.array(want))) <= 1e-12


def all_pin_checks(golden_dir):
    return [
        check_storage_f16,
        check_storage_bf16,
        lambda: check_golden_velog(golden_dir),
        lambda: check_golden_digest(golden_dir),
        lambda: check_golden_on_demand(golden_dir),
        check_brute_force_tiny,
        lambda: check_sdpa_library("f32"),
        lambda: check_sdpa_library("f16"),
        lambda: check_sdpa_library("bf16"),
        check_one_token_returns_v,
        check_zero_query_gives_mean,
        check_two_tokens_logistic,
        check_dominant_key,
        check_empty_context_zero,
        check_permutation_invariance,
        check_block_size_invariance,
        check_append_brute_force,
        check_block_copy_brute_force,
        check_gqa_equals_replicated_mha,
        check_multi_query_rows_are_shorter_decodes,
    ]


# ---------------------------------------------------------------------------
# Tests
# ---------------------------------------------------------------------------

def test_storage_f16():
    check_storage_f16()


def test_storage_bf16():
    check_storage_bf16()


def test_golden_velog_table(golden_dir):
    check_golden_velog(golden_dir)


def test_golden_digest_flowchart(golden_dir):
    check_golden_digest(golden_dir)


def test_golden_on_demand_allocation(golden_dir):
    check_golden_on_demand(golden_dir)


def test_brute_force_tiny():
    check_brute_force_tiny()


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_library_attention(dtype):
    check_sdpa_library(dtype)


def test_one_token_returns_v():
    check_one_token_returns_v()


def test_zero_query_gives_mean():
    check_zero_query_gives_mean()


def test_two_tokens_logistic():
    check_two_tokens_logistic()


def test_dominant_key():
    check_dominant_key()


def test_empty_context_zero():
    check_empty_context_zero()


def test_permutation_invariance():
    check_permutation_invariance()


def test_block_size_invariance():
    check_block_size_invariance()


def test_append_brute_force():
    check_append_brute_force()


def test_block_copy_brute_force():
    check_block_copy_brute_force()


def test_gqa_equals_replicated_mha():
    check_gqa_equals_replicated_mha()


def test_multi_query_rows_are_shorter_decodes():
    check_multi_query_rows_are_shorter_decodes()


def test_softmax_weights_sum_to_one():
    rng = np.random.default_rng(21)
    for n in (1, 2, 7, 1000):
        w = oracle.softmax_weights(rng.standard_normal(n) * 30)
        assert abs(math.fsum(w) - 1.0) < 1e-12 and np.all(w >= 0)


# ---- planted mistakes -------------------------------------------------------

_orig_gather_rows = paged_attention.gather_rows
_orig_attend = paged_attention.attend
_orig_softmax = paged_attention.softmax_weights


def _mut_block_off_by_one(pool, table_row, ctx, head, block_size):
    t = np.arange(int(ctx))
    phys = np.asarray(table_row)[np.minimum((t + 1) // block_size, len(table_row) - 1)]
    return pool[np.maximum(phys, 0), head, t % block_size, :]


def _mut_div_mod_swapped(pool, table_row, ctx, head, block_size):
    t = np.arange(int(ctx))
    idx = np.minimum(t % block_size, len(table_row) - 1)
    phys = np.maximum(np.asarray(table_row)[idx], 0)
    return pool[phys, head, (t // block_size) % block_size, :]


def _mut_mask_short(pool, table_row, ctx, head, block_size):
    return _orig_gather_rows(pool, table_row, max(int(ctx) - 1, 0) if ctx > 1 else ctx, head, block_size)


def _mut_gqa_head_modulo(q, k_pool, v_pool, block_tables, context_lens, scale, block_size, dtype, selection):
    """Reads K/V head h % Hkv instead of h // G (a plausible grouping mistake)."""
    Hkv = k_pool.shape[1]
    D = q.shape[2]
    out = np.zeros((len(selection), D))
    for i, (s, h) in enumerate(selection):
        ctx = int(context_lens[s])
        K = storage.to_f64(_orig_gather_rows(k_pool, block_tables[s], ctx, h % Hkv, block_size), dtype)
        V = storage.to_f64(_orig_gather_rows(v_pool, block_tables[s], ctx, h % Hkv, block_size), dtype)
        out[i] = _orig_attend(storage.to_f64(q[s, h], dtype), K, V, scale)
    return out


def _mut_no_scale(q, K, V, scale):
    return _orig_attend(q, K, V, 1.0)


def _mut_kv_swapped(q, K, V, scale):
    return _orig_attend(q, V, K, scale)


def _mut_neg_logits(logits):
    return _orig_softmax(-np.asarray(logits, dtype=np.float64))


def _mut_append_div_mod_swapped(k_pool, v_pool, k_new, v_new, slot_mapping, block_size):
    nb = k_pool.shape[0]
    swapped = [(s % block_size) * block_size + (s // block_size) % block_size if s >= 0 else s
               for s in np.asarray(slot_mapping).tolist()]
    swapped = [s if s < nb * block_size else -1 for s in swapped]
    return _orig_append(k_pool, v_pool, k_new, v_new, np.array(swapped), block_size)


def _mut_copy_k_only(k_pool, v_pool, pairs):
    k, _, bad = _orig_copy(k_pool, v_pool, pairs)
    return k, np.array(v_pool, copy=True), bad


_orig_append = cache_ops.kv_append
_orig_copy = cache_ops.kv_block_copy


MUTANTS = {
    "block index off by one": [(paged_attention, "gather_rows", _mut_block_off_by_one)],
    "block/slot div-mod swapped": [(paged_attention, "gather_rows", _mut_div_mod_swapped)],
    "context mask one short": [(paged_attention, "gather_rows", _mut_mask_short)],
    "scale dropped": [(paged_attention, "attend", _mut_no_scale)],
    "K and V swapped": [(paged_attention, "attend", _mut_kv_swapped)],
    "logit sign flipped": [(paged_attention, "softmax_weights", _mut_neg_logits)],
    "bf16 decoded as fp16": [(storage, "to_f64", "bf16_as_f16")],
    "append block/offset swapped": [(cache_ops, "kv_append", _mut_append_div_mod_swapped)],
    "block copy forgets V": [(cache_ops, "kv_block_copy", _mut_copy_k_only)],
    "query head grouped by modulo": [(paged_attention, "paged_decode_selected", _mut_gqa_head_modulo)],
}


def _apply(monkeypatch, patches):
    import oracle as pkg
    from oracle import paged_attention as pa_mod
    for mod, name, repl in patches:
        if repl == "bf16_as_f16":
            orig = storage.to_f64

            def repl(raw, dtype, _orig=orig):
                return _orig(raw, "f16" if dtype == "bf16" else dtype)
        monkeypatch.setattr(mod, name, repl)
        if hasattr(pkg, name):
            monkeypatch.setattr(pkg, name, repl)
        if mod is storage:
            monkeypatch.setattr(pa_mod, name, repl)


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistakes_are_caught(mutant, monkeypatch, golden_dir):
    _apply(monkeypatch, MUTANTS[mutant])
    failures = 0
    for check in all_pin_checks(golden_dir):
        try:
            check()
        except Exception:
            failures += 1
    assert failures >= 1, f"no pin caught the planted mistake: {mutant}"


def test_pins_pass_unmutated(golden_dir):
    for check in all_pin_checks(golden_dir):
        check()
