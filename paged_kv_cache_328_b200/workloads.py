"""Seeded synthetic inputs for paged decode attention and the cache operations.

This module only *builds inputs*: random lengths, a random placement of logical
blocks in the physical pool, block tables, slot mappings for the step's new
token, copy-on-write pairs, and N(0,1) values for q, K and V.  It holds none of
the attention, append or copy arithmetic; the CUDA library and the CPU oracle
both consume what it returns.

Conventions shared by every workload:

* Pools are ``[num_blocks, H, B, D]`` in the storage dtype; unused blocks and the
  slots past each sequence's context are filled with NaN so that any stray read
  shows up in the output.
* ``context_lens[s]`` is the number of tokens attended in this step, i.e. it
  already counts the token appended in this step (compute the new K/V, add it
  to the cache, then attend: "LLM Inference 8 - PagedAttention", section
  "KV Cache의 메모리 문제").  The appended token of sequence s sits at logical
  position ``context_lens[s] - 1``; ``slot_mapping[s]`` addresses it, or is -1
  when the context is empty.
* Blocks are taken on demand, ``ceil(ctx / B)`` per sequence, and the
  block table is padded with -1 ("LLM Inference 8 - PagedAttention", section
  "PagedAttention의 동작 방식").
* With ``preappend=True`` the pool holds the context *without* the step's token
  (its slot is NaN) so that the append must happen before the attention reads it.

Workload shapes follow the five configurations of the hot-path specification:
``tiny``, ``llama7b``, ``opt13b``, ``cow`` and ``longctx`` (seed 3280 + index).
"""

from dataclasses import dataclass, field
import math

import numpy as np
import torch

TORCH_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}

CONFIG_INDEX = {"tiny": 1, "llama7b": 2, "opt13b": 3, "cow": 4, "longctx": 5}
BASE_SEED = 3280


@dataclass
class Workload:
    name: str
    S: int
    H: int
    D: int
    B: int
    dtype: str
    scale: float
    num_blocks: int
    max_blocks: int
    context_lens: np.ndarray          # int32 [S], tokens attended this step
    block_tables: np.ndarray          # int32 [S, max_blocks], -1 padded
    slot_mapping: np.ndarray          # int64 [T], slot of each appended token (-1 = none)
    cow_pairs: np.ndarray             # int64 [n, 2] (src, dst) block copies of the step
    q: torch.Tensor                   # [S, H, D] storage dtype
    k_pool: torch.Tensor              # [NB, H, B, D]
    v_pool: torch.Tensor
    k_new: torch.Tensor               # [T, H, D], the step's appended rows
    v_new: torch.Tensor
    partition_tokens: int = 0         # split-context partition size (0 = library default)
    info: dict = field(default_factory=dict)
    Hkv: int = 0                      # K/V heads in the pools (0: same as H, multi-head)

    def __post_init__(self):
        if not self.Hkv:
            self.Hkv = self.H

    # ---- sizes -------------------------------------------------------------
    @property
    def elem_bytes(self):
        return ELEM_BYTES[self.dtype]

    def kv_bytes_attended(self):
        """K+V bytes the decode reads by definition: sum(ctx) * Hkv * D * e * 2."""
        return int(self.context_lens.astype(np.int64).sum()) * self.Hkv * self.D * self.elem_bytes * 2

    def append_bytes(self):
        n = int((self.slot_mapping >= 0).sum())
        return n * self.Hkv * self.D * self.elem_bytes * 2

    def copy_bytes(self):
        """K+V bytes read (equal to bytes written) by the step's block copies."""
        return len(self.cow_pairs) * self.Hkv * self.B * self.D * self.elem_bytes * 2

    # ---- host views (raw stored elements) ------------------------------------
    def host(self, t):
        """Stored elements of a tensor as NumPy: float32, or uint16 bit patterns."""
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.float32:
            return t.numpy()
        return t.view(torch.int16).numpy().view(np.uint16)


def _nan_pool(nb, H, B, D, dtype, device):
    return torch.full((nb, H, B, D), float("nan"), dtype=TORCH_DTYPES[dtype], device=device)


def _randn(shape, gen, dtype, device, chunk_rows=1 << 14):
    """N(0,1) values drawn in fp32 from ``gen`` (row chunks bound the fp32 temporaries), cast."""
    out = torch.empty(shape, dtype=TORCH_DTYPES[dtype], device=device)
    rows = shape[0]
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen,
                                 dtype=torch.float32, device=device).to(out.dtype)
    return out


def _scatter_tokens(pool, phys, off, rows, chunk=1 << 16):
    """pool[phys[i], :, off[i], :] = rows[i] (placement of logical rows into their slots)."""
    by_slot = pool.permute(0, 2, 1, 3)  # view [NB, B, H, D]
    for i0 in range(0, len(phys), chunk):
        i1 = min(len(phys), i0 + chunk)
        by_slot[phys[i0:i1], off[i0:i1]] = rows[i0:i1]


def _token_coords(tables, ctx, B, device, skip_last):
    """Physical (block, slot) of every stored logical token, sequence-major order."""
    phys, off = [], []
    for s, c in enumerate(ctx.tolist()):
        n = c - 1 if (skip_last and c > 0) else c
        if n <= 0:
            continue
        t = np.arange(n)
        phys.append(tables[s, t // B].astype(np.int64))
        off.append((t % B).astype(np.int64))
    if not phys:
        z = torch.zeros(0, dtype=torch.long, device=device)
        return z, z
    return (torch.from_numpy(np.concatenate(phys)).to(device),
            torch.from_numpy(np.concatenate(off)).to(device))


def build_paged(context_lens, H, D, B, dtype, seed, *, device="cpu", num_blocks=None,
                pool_factor=1.2, max_blocks=None, preappend=False, scale=None,
                placement_seed=None, name="custom", partition_tokens=0, logical=None,
                num_q_heads=None):
    """Independent sequences with a random physical placement of their blocks.

    ``H`` is the number of K/V heads in the pools; ``num_q_heads`` (default H)
    the number of query heads, a multiple of H (grouped-query attention).
    ``logical`` may pass pre-drawn per-token rows ``(K_log, V_log, q)`` with
    ``K_log``/``V_log`` of shape ``[sum(ctx), H, D]`` so that several block sizes
    share the same token data; otherwise they are drawn from ``seed``.
    """
    Hq = H if num_q_heads is None else int(num_q_heads)
    if Hq % H:
        raise ValueError("query heads must be a multiple of K/V heads")
    ctx = np.asarray(context_lens, dtype=np.int64)
    S = len(ctx)
    nblk = -(-ctx // B)
    needed = int(nblk.sum())
    if num_blocks is None:
        num_blocks = max(1, int(math.ceil(pool_factor * needed)))
    if num_blocks < needed:
        raise ValueError("pool too small for the contexts")
    if max_blocks is None:
        max_blocks = max(1, int(nblk.max()) if S else 1)
    if int(nblk.max(initial=0)) > max_blocks:
        raise ValueError("a context needs more than max_blocks blocks")

    prng = np.random.default_rng(seed if placement_seed is None else placement_seed)
    perm = prng.permutation(num_blocks)
    tables = np.full((S, max_blocks), -1, dtype=np.int32)
    cursor = 0
    for s in range(S):
        n = int(nblk[s])
        tables[s, :n] = perm[cursor:cursor + n]
        cursor += n

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    total = int(ctx.sum())
    if logical is None:
        K_log = _randn((total, H, D), gen, dtype, device)
        V_log = _randn((total, H, D), gen, dtype, device)
        q = _randn((S, Hq, D), gen, dtype, device)
    else:
        K_log, V_log, q = logical

    starts = np.concatenate([[0], np.cumsum(ctx)[:-1]]).astype(np.int64) if S else np.zeros(0, np.int64)
    keep = []
    for s in range(S):
        n = int(ctx[s]) - 1 if (preappend and ctx[s] > 0) else int(ctx[s])
        keep.append(np.arange(starts[s], starts[s] + n))
    keep = torch.from_numpy(np.concatenate(keep) if keep else np.zeros(0, np.int64)).to(device)
    phys, off = _token_coords(tables, ctx, B, device, skip_last=preappend)

    k_pool = _nan_pool(num_blocks, H, B, D, dtype, device)
    v_pool = _nan_pool(num_blocks, H, B, D, dtype, device)
    if len(keep):
        _scatter_tokens(k_pool, phys, off, K_log.index_select(0, keep))
        _scatter_tokens(v_pool, phys, off, V_log.index_select(0, keep))

    slot = np.full(S, -1, dtype=np.int64)
    last = np.zeros(S, dtype=np.int64)
    for s in range(S):
        c = int(ctx[s])
        if c > 0:
            pos = c - 1
            slot[s] = int(tables[s, pos // B]) * B + pos % B
            last[s] = starts[s] + pos
    if total > 0:
        lastt = torch.from_numpy(last).to(device)
        k_new = K_log.index_select(0, lastt)
        v_new = V_log.index_select(0, lastt)
    else:  # no context holds a token: nothing to append (every slot is -1)
        k_new = torch.zeros((S, H, D), dtype=K_log.dtype, device=device)
        v_new = torch.zeros((S, H, D), dtype=V_log.dtype, device=device)

    return Workload(
        name=name, S=S, H=Hq, D=D, B=B, dtype=dtype, Hkv=H,
        scale=(1.0 / math.sqrt(D)) if scale is None else float(scale),
        num_blocks=num_blocks, max_blocks=max_blocks,
        context_lens=ctx.astype(np.int32), block_tables=tables, slot_mapping=slot,
        cow_pairs=np.zeros((0, 2), dtype=np.int64),
        q=q, k_pool=k_pool, v_pool=v_pool, k_new=k_new, v_new=v_new,
        partition_tokens=partition_tokens,
        info={"seed": seed, "blocks_used": needed},
    )


def draw_logical(total_tokens, S, H, D, dtype, seed, device):
    """Per-token K/V rows and q drawn once, to place the same tokens under several block sizes."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    K_log = _randn((total_tokens, H, D), gen, dtype, device)
    V_log = _randn((total_tokens, H, D), gen, dtype, device)
    q = _randn((S, H, D), gen, dtype, device)
    return K_log, V_log, q


# ---------------------------------------------------------------------------
# Context-length distributions of the five configurations
# ---------------------------------------------------------------------------

def tiny_lengths():
    """Tiny case: contexts {1, 15, 16, 37} before the step's append, {2, 16, 17, 38} after."""
    return np.array([2, 16, 17, 38], dtype=np.int64)


def lognormal_lengths(S, seed, mean=340.0, sigma=1.0, lo=1, hi=2048):
    """Lognormal with arithmetic mean ``mean`` and log-space sd ``sigma``, rounded and clipped."""
    rng = np.random.default_rng(seed)
    mu = math.log(mean) - sigma * sigma / 2.0
    x = np.rint(rng.lognormal(mu, sigma, size=S)).astype(np.int64)
    return np.clip(x, lo, hi)


def uniform_lengths(S, seed, lo, hi):
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=S).astype(np.int64)


def make_tiny(device="cpu", preappend=True):
    """4 sequences, 2 heads x 64, fp32, B=16 in a 16-block pool; plus one CoW pair."""
    seed = BASE_SEED + CONFIG_INDEX["tiny"]
    w = build_paged(tiny_lengths(), H=2, D=64, B=16, dtype="f32", seed=seed, device=device,
                    num_blocks=16, preappend=preappend, scale=1.0 / 8.0, name="tiny")
    used = set(w.block_tables[w.block_tables >= 0].tolist())
    free = [b for b in range(w.num_blocks) if b not in used]
    rng = np.random.default_rng(seed + 1)
    dst = int(rng.choice(free))
    src = int(w.block_tables[3, (int(w.context_lens[3]) - 1) // w.B])
    w.cow_pairs = np.array([[src, dst]], dtype=np.int64)
    return w


def make_llama7b(device="cpu", preappend=False, S=64):
    seed = BASE_SEED + CONFIG_INDEX["llama7b"]
    ctx = lognormal_lengths(S, seed)
    return build_paged(ctx, H=32, D=128, B=16, dtype="f16", seed=seed, device=device,
                       preappend=preappend, max_blocks=2048 // 16, name="llama7b")


def opt13b_lengths(S=256):
    return uniform_lengths(S, BASE_SEED + CONFIG_INDEX["opt13b"], 1, 2048)


def make_opt13b(B=16, device="cpu", preappend=False, S=256, logical=None):
    """Batch-256 OPT-13B decode layer; the token data is the same for every B."""
    seed = BASE_SEED + CONFIG_INDEX["opt13b"]
    ctx = opt13b_lengths(S)
    if logical is None:
        logical = draw_logical(int(ctx.sum()), S, 40, 128, "bf16", seed, device)
    return build_paged(ctx, H=40, D=128, B=B, dtype="bf16", seed=seed, device=device,
                       preappend=preappend, max_blocks=2048 // B, logical=logical,
                       placement_seed=seed * 1000 + B, name=f"opt13b_B{B}")


def make_longctx(device="cpu", preappend=False, S=8, partition_tokens=512):
    seed = BASE_SEED + CONFIG_INDEX["longctx"]
    ctx = uniform_lengths(S, seed, 16384, 32768)
    return build_paged(ctx, H=40, D=128, B=16, dtype="f16", seed=seed, device=device,
                       preappend=preappend, max_blocks=32768 // 16,
                       partition_tokens=partition_tokens, name="longctx")


def make_cow(device="cpu", preappend=False, groups=32, n=4, prompt=512, tail_max=256,
             H=40, D=128, B=16, dtype="f16"):
    """Parallel sampling: ``groups`` prompts of ``prompt`` tokens, ``n`` samples per prompt.

    The prompt blocks of a group are stored once and shared by its n samples (the
    block manager's reference count is n).  Each sample owns a private tail of
    U{1..tail_max} generated tokens plus the token appended this step.  Reading
    of "CoW of the shared partial block": every step each non-owner sample
    writes into its own copy of the group's last prompt block, so the step forks
    that block once per non-owner sample ((n-1) * groups pairs, src = shared
    block, dst = a fresh block) and those samples' tables point at their copies.
    """
    seed = BASE_SEED + CONFIG_INDEX["cow"]
    rng = np.random.default_rng(seed)
    if prompt % B:
        raise ValueError("prompt must fill whole blocks")
    pb = prompt // B
    S = groups * n
    tails = rng.integers(1, tail_max + 1, size=S).astype(np.int64)
    ctx = prompt + tails + 1
    tail_blocks = -(-(tails + 1) // B)
    needed = groups * pb + (n - 1) * groups + int(tail_blocks.sum())
    num_blocks = int(math.ceil(1.2 * needed))
    max_blocks = pb + int(-(-(tail_max + 1) // B))
    perm = rng.permutation(num_blocks)
    cur = 0

    def take(k):
        nonlocal cur
        out = perm[cur:cur + k]
        cur += k
        return out

    tables = np.full((S, max_blocks), -1, dtype=np.int32)
    pairs = []
    shared = []
    for g in range(groups):
        blocks = take(pb)
        shared.append(blocks)
        for i in range(n):
            s = g * n + i
            tables[s, :pb] = blocks
            if i > 0:
                dst = int(take(1)[0])
                tables[s, pb - 1] = dst
                pairs.append((int(blocks[pb - 1]), dst))
            tables[s, pb:pb + tail_blocks[s]] = take(int(tail_blocks[s]))

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    P_K = _randn((groups * prompt, H, D), gen, dtype, device)
    P_V = _randn((groups * prompt, H, D), gen, dtype, device)
    T_K = _randn((int((tails + 1).sum()), H, D), gen, dtype, device)
    T_V = _randn((int((tails + 1).sum()), H, D), gen, dtype, device)
    q = _randn((S, H, D), gen, dtype, device)

    k_pool = _nan_pool(num_blocks, H, B, D, dtype, device)
    v_pool = _nan_pool(num_blocks, H, B, D, dtype, device)
    # shared prompt tokens: stored once per group, in the group's shared blocks
    t = np.arange(prompt)
    ph = np.concatenate([shared[g][t // B] for g in range(groups)]).astype(np.int64)
    of = np.tile(t % B, groups).astype(np.int64)
    _scatter_tokens(k_pool, torch.from_numpy(ph).to(device), torch.from_numpy(of).to(device), P_K)
    _scatter_tokens(v_pool, torch.from_numpy(ph).to(device), torch.from_numpy(of).to(device), P_V)
    # private tails (the step's token is left out when preappend)
    tstarts = np.concatenate([[0], np.cumsum(tails + 1)[:-1]]).astype(np.int64)
    ph, of, rows, slot, last = [], [], [], np.full(S, -1, np.int64), np.zeros(S, np.int64)
    for s in range(S):
        nt = int(tails[s]) + (0 if preappend else 1)
        pos = prompt + np.arange(nt)
        ph.append(tables[s, pos // B].astype(np.int64))
        of.append((pos % B).astype(np.int64))
        rows.append(tstarts[s] + np.arange(nt))
        p = prompt + int(tails[s])
        slot[s] = int(tables[s, p // B]) * B + p % B
        last[s] = tstarts[s] + int(tails[s])
    ph = torch.from_numpy(np.concatenate(ph)).to(device)
    of = torch.from_numpy(np.concatenate(of)).to(device)
    rows = torch.from_numpy(np.concatenate(rows)).to(device)
    _scatter_tokens(k_pool, ph, of, T_K.index_select(0, rows))
    _scatter_tokens(v_pool, ph, of, T_V.index_select(0, rows))
    lastt = torch.from_numpy(last).to(device)

    unique = groups * pb + int(tail_blocks.sum())
    unshared = int((pb + tail_blocks).sum())
    return Workload(
        name="cow", S=S, H=H, D=D, B=B, dtype=dtype, scale=1.0 / math.sqrt(D),
        num_blocks=num_blocks, max_blocks=max_blocks,
        context_lens=ctx.astype(np.int32), block_tables=tables, slot_mapping=slot,
        cow_pairs=np.array(pairs, dtype=np.int64).reshape(-1, 2),
        q=q, k_pool=k_pool, v_pool=v_pool,
        k_new=T_K.index_select(0, lastt), v_new=T_V.index_select(0, lastt),
        info={"seed": seed, "blocks_used": needed,
              "blocks_shared_layout": unique, "blocks_if_unshared": unshared,
              "cow_saving": 1.0 - unique / unshared},
    )


def make_gqa(group, device="cpu", preappend=False, S=256, Hkv=8, B=16):
    """Grouped-query decode layer: 8 K/V heads x 128 (bf16) shared by `group` query heads
    each, batch 256, contexts U{1..2048} (the batch-256 layer's lengths), block size 16."""
    seed = BASE_SEED + 10 + group
    ctx = opt13b_lengths(S)
    return build_paged(ctx, H=Hkv, D=128, B=B, dtype="bf16", seed=seed, device=device, preappend=preappend,
                       max_blocks=2048 // B, num_q_heads=Hkv * group, name=f"gqa{group}_B{B}")


def make(name, device="cpu", preappend=False, B=None):
    if name == "tiny":
        return make_tiny(device=device, preappend=preappend)
    if name == "llama7b":
        return make_llama7b(device=device, preappend=preappend)
    if name == "opt13b":
        return make_opt13b(B=16 if B is None else B, device=device, preappend=preappend)
    if name == "cow":
        return make_cow(device=device, preappend=preappend)
    if name == "longctx":
        return make_longctx(device=device, preappend=preappend)
    if name.startswith("gqa"):
        return make_gqa(int(name[3:]), device=device, preappend=preappend, B=16 if B is None else B)
    raise ValueError(f"unknown workload {name!r}")


def last_block_waste(w):
    """Fraction of reserved slots left empty: only each sequence's last block is partial."""
    from .tuning import last_block_waste as waste
    return waste(w.context_lens, w.B)
