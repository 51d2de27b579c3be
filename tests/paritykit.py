"""Helpers for the GPU parity tests: device copies of workload indices, and
host-side snapshots of the blocks a sampled (sequence, head) needs, taken
before any library kernel runs so that the oracle's inputs never come from the
CUDA path."""

import numpy as np
import torch

import oracle

TOL = {"f32": 1e-5, "f16": 2e-3, "bf16": 2e-3}


def dev_indices(w, device):
    return dict(
        bt=torch.from_numpy(w.block_tables).to(device),
        ctx=torch.from_numpy(w.context_lens).to(device),
        slots=torch.from_numpy(w.slot_mapping).to(device),
        pairs=torch.from_numpy(w.cow_pairs.reshape(-1, 2)).to(device),
    )


class Snapshot:
    """Pre-step host copy of what one (sequence, head) reads, remapped to a compact pool."""

    def __init__(self, w, s, h):
        self.s, self.h = s, h
        kvh = h // (w.H // w.Hkv)  # K/V head read by query head h
        ctx = int(w.context_lens[s])
        nblk = -(-ctx // w.B)
        row = [int(b) for b in w.block_tables[s, :nblk]]
        srcs = [int(a) for a, b in w.cow_pairs.reshape(-1, 2).tolist() if b in row]
        blocks = sorted(set(row) | set(srcs))
        self.remap = {b: i for i, b in enumerate(blocks)}
        idx = torch.tensor(blocks, dtype=torch.long, device=w.k_pool.device)
        self.k = w.host(w.k_pool.index_select(0, idx)[:, kvh:kvh + 1].contiguous())
        self.v = w.host(w.v_pool.index_select(0, idx)[:, kvh:kvh + 1].contiguous())
        self.table = np.array([self.remap[b] for b in row], dtype=np.int64).reshape(1, -1)
        if nblk == 0:
            self.table = np.full((1, 1), -1, dtype=np.int64)
        self.pairs = np.array([[self.remap[a], self.remap[b]] for a, b in w.cow_pairs.reshape(-1, 2).tolist()
                               if b in self.remap], dtype=np.int64).reshape(-1, 2)
        slot = int(w.slot_mapping[s])
        if slot >= 0:
            blk, off = divmod(slot, w.B)
            self.slot = np.array([self.remap[blk] * w.B + off], dtype=np.int64)
        else:
            self.slot = np.array([-1], dtype=np.int64)
        self.q = w.host(w.q[s:s + 1, h:h + 1].contiguous())
        self.knew = w.host(w.k_new[s:s + 1, kvh:kvh + 1].contiguous()) if w.k_new.shape[0] > s else None
        self.vnew = w.host(w.v_new[s:s + 1, kvh:kvh + 1].contiguous()) if w.v_new.shape[0] > s else None
        self.ctx = ctx

    def expected(self, w, copy=True, append=True, ctx=None):
        """Oracle output of this (sequence, head) after the step's copy and append."""
        k, v = self.k, self.v
        if copy and len(self.pairs):
            k, v, bad = oracle.kv_block_copy(k, v, self.pairs)
            assert bad == 0
        if append and self.knew is not None and self.slot[0] >= 0:
            k, v, bad = oracle.kv_append(k, v, self.knew, self.vnew, self.slot, w.B)
            assert bad == 0
        c = self.ctx if ctx is None else ctx
        return oracle.paged_decode(self.q, k, v, self.table, np.array([c]), w.scale, w.B, w.dtype)[0, 0]


def sample_pairs(w, n, seed):
    rng = np.random.default_rng(seed)
    sel = set()
    # always include the longest and the shortest contexts
    sel.add((int(np.argmax(w.context_lens)), int(rng.integers(w.H))))
    sel.add((int(np.argmin(w.context_lens)), int(rng.integers(w.H))))
    while len(sel) < n:
        sel.add((int(rng.integers(w.S)), int(rng.integers(w.H))))
    return sorted(sel)


def max_err(got, want):
    got = np.asarray(got, dtype=np.float64)
    return float(np.max(np.abs(got - want))) if got.size else 0.0
