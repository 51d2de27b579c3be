"""The C-ABI library: it builds, loads without a GPU, exports every declared symbol,
and rejects bad arguments on the host before any CUDA call (no GPU needed)."""

import ctypes
import os
import re

import pytest

from conftest import ROOT
from paged_kv_cache_328_b200 import _lib
from paged_kv_cache_328_b200 import build as builder

HEADER = os.path.join(ROOT, "include", "pagedkv.h")

PKV_OK, PKV_EINVAL, PKV_EDTYPE, PKV_EALIGN, PKV_EUNSUPPORTED = 0, -1, -2, -3, -4
PKV_EWORKSPACE = -6


@pytest.fixture(scope="module")
def lib():
    builder.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("paged_attn_decode", "kv_cache_append", "kv_block_copy", "paged_attn_decode_workspace_size",
              "pkv_get_device_error", "pkv_strerror", "paged_kv_gather"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_library_is_built_for_sm100a_only(lib):
    # the build command is the contract: one gencode, sm_100a
    assert builder.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert os.path.exists(builder.LIB)


def test_strerror_and_version(lib):
    assert _lib.abi_version() == 1
    for code in range(-8, 1):
        assert _lib.strerror(code) != "unknown error code"
    assert _lib.strerror(-99) == "unknown error code"


def test_workspace_size_layout(lib):
    # no split: counters (16) + an 8-byte unit entry per sequence, rounded to 16
    assert _lib.workspace_size(256, 40, 128, 16, 128, 2048) == 16 + 2048
    # split into 64 partitions of 512 tokens: + m/l and acc per partition
    n = _lib.workspace_size(8, 40, 128, 16, 2048, 512)
    assert n == 16 + 8 * 64 * 8 + 8 * 40 * 64 * 8 + 8 * 40 * 64 * 128 * 4
    assert _lib.partition_tokens(8, 40, 128, 16, 2048, 512) == 512
    # the library's own choice splits long contexts into 512-token partitions
    assert _lib.partition_tokens(8, 40, 128, 16, 2048, 0) == 512
    # a partition as long as the longest context means no split
    assert _lib.partition_tokens(4, 2, 64, 16, 3, 0) == 48
    # enough (sequence, head) pairs and contexts <= 4096: no split by default
    assert _lib.partition_tokens(256, 40, 128, 16, 128, 0) == 2048
    assert _lib.partition_tokens(64, 32, 128, 16, 128, 0) == 2048     # 2048 pairs: no split
    assert _lib.partition_tokens(32, 32, 128, 16, 128, 0) == 512      # 1024 pairs: split
    assert _lib.partition_tokens(256, 40, 128, 16, 512, 0) == 512     # contexts up to 8192: split


@pytest.mark.parametrize("args, code", [
    ((4, 2, 64, 16, 3, 24), PKV_EINVAL),        # not a multiple of B
    ((4, 2, 64, 16, 3, -16), PKV_EINVAL),
    ((4, 2, 96, 16, 3, 0), PKV_EUNSUPPORTED),   # head_dim
    ((4, 2, 64, 12, 3, 0), PKV_EUNSUPPORTED),   # block_size
    ((-1, 2, 64, 16, 3, 0), PKV_EINVAL),
    ((70000, 2, 64, 16, 3, 0), PKV_EINVAL),
    ((4, 0, 64, 16, 3, 0), PKV_EINVAL),
])
def test_partition_rejections(lib, args, code):
    assert lib.paged_attn_decode_partition_tokens(*args) == code
    assert lib.paged_attn_decode_workspace_size(*args) == ctypes.c_size_t(-1).value


A = 0x10000  # an aligned fake device address; rejected calls never dereference it


def decode_args(**over):
    a = dict(q=A, k=A, v=A, bt=A, cl=A, S=4, H=2, D=64, B=16, MB=3, NB=16, dt=0, scale=0.125, out=A,
             pt=0, ws=A, wsb=1 << 20, stream=None)
    a.update(over)
    return [a[k] for k in ("q", "k", "v", "bt", "cl", "S", "H", "D", "B", "MB", "NB", "dt", "scale", "out",
                           "pt", "ws", "wsb", "stream")]


@pytest.mark.parametrize("over, code", [
    (dict(q=None), PKV_EINVAL),
    (dict(out=None), PKV_EINVAL),
    (dict(bt=None), PKV_EINVAL),
    (dict(q=A + 8), PKV_EALIGN),
    (dict(k=A + 4), PKV_EALIGN),
    (dict(out=A + 4), PKV_EALIGN),
    (dict(cl=A + 2), PKV_EALIGN),
    (dict(ws=A + 8), PKV_EALIGN),
    (dict(dt=7), PKV_EDTYPE),
    (dict(D=80), PKV_EUNSUPPORTED),
    (dict(B=24), PKV_EUNSUPPORTED),
    (dict(pt=8), PKV_EINVAL),
    (dict(NB=0), PKV_EINVAL),
    (dict(scale=float("nan")), PKV_EINVAL),
    (dict(wsb=16), PKV_EWORKSPACE),
])
def test_decode_rejects_on_host(lib, over, code):
    assert lib.paged_attn_decode(*decode_args(**over)) == code


def test_decode_empty_batch_is_a_no_op(lib):
    assert lib.paged_attn_decode(*decode_args(S=0)) == PKV_OK


def test_append_and_copy_reject_on_host(lib):
    # kv_cache_append(k, v, kc, vc, slots, T, H, D, B, NB, dt, stream)
    assert lib.kv_cache_append(A, A, A, A, A, 0, 2, 64, 16, 4, 0, None) == PKV_OK          # nothing to do
    assert lib.kv_cache_append(None, A, A, A, A, 1, 2, 64, 16, 4, 0, None) == PKV_EINVAL
    assert lib.kv_cache_append(A, A, A, A, A + 4, 1, 2, 64, 16, 4, 0, None) == PKV_EALIGN
    assert lib.kv_cache_append(A, A, A, A, A, 1, 2, 48, 16, 4, 0, None) == PKV_EUNSUPPORTED
    assert lib.kv_cache_append(A, A, A, A, A, -1, 2, 64, 16, 4, 0, None) == PKV_EINVAL
    assert lib.kv_cache_append(A, A, A, A, A, 1, 2, 64, 16, 4, 3, None) == PKV_EDTYPE
    # kv_block_copy(kc, vc, pairs, n, H, D, B, NB, dt, stream)
    assert lib.kv_block_copy(A, A, A, 0, 2, 64, 16, 4, 0, None) == PKV_OK
    assert lib.kv_block_copy(A, A, None, 1, 2, 64, 16, 4, 0, None) == PKV_EINVAL
    assert lib.kv_block_copy(A, A + 8, A, 1, 2, 64, 16, 4, 0, None) == PKV_EALIGN
    assert lib.kv_block_copy(A, A, A, 1, 2, 64, 17, 4, 0, None) == PKV_EUNSUPPORTED
    # paged_kv_gather(cache, table, ctx, H, D, B, NB, dt, out, stream)
    assert lib.paged_kv_gather(A, A, 0, 2, 64, 16, 4, 0, A, None) == PKV_OK
    assert lib.paged_kv_gather(A, A, -1, 2, 64, 16, 4, 0, A, None) == PKV_EINVAL
    assert lib.paged_kv_gather(A, A, 5, 2, 64, 16, 4, 0, A + 8, None) == PKV_EALIGN


def test_binding_refuses_cpu_tensors(lib):
    import torch
    q = torch.zeros(1, 2, 64)
    kc = torch.zeros(4, 2, 16, 64)
    with pytest.raises(ValueError, match="CUDA"):
        _lib.paged_attn_decode(q, kc, kc, torch.zeros(1, 1, dtype=torch.int32),
                               torch.zeros(1, dtype=torch.int32), 1.0,
                               workspace=torch.zeros(64, dtype=torch.uint8))


def test_wait_selftest_rejects_limits_on_host(lib):
    assert lib.pkv_selftest_wait_timeout(0, None) == PKV_EINVAL
    assert lib.pkv_selftest_wait_timeout(-5, None) == PKV_EINVAL
    assert lib.pkv_selftest_wait_timeout(2_000_000_001, None) == PKV_EINVAL


def test_multi_query_plan_counts_128_row_tiles_above_16_rows(lib):
    # 32 query rows per K/V head (Lq = 32, G = 1) run on the tcgen05 kernel's 128-row tiles:
    # 100 sequences x 8 K/V heads x 1 tile = 800 units < 4 x 296, so contexts up to 2048 are split
    # into 512-token partitions (with 16-row tiles it would be 1600 units and no split)
    S, Lq, H, Hkv, D, B, MB = 100, 32, 8, 8, 128, 16, 128
    P, rows = 4, Lq * H
    split = 16 + S * P * 8 + S * rows * P * 8 + S * rows * P * D * 4
    assert lib.paged_attn_multi_query_workspace_size(S, Lq, H, Hkv, D, B, MB, 0) == split
    # 16 rows per K/V head (Lq = 2, G = 8) stay on 16-row tiles: 800 units as well, split
    P, rows = 4, 2 * 64
    assert lib.paged_attn_multi_query_workspace_size(S, 2, 64, 8, D, B, MB, 0) == \
        16 + S * P * 8 + S * rows * P * 8 + S * rows * P * D * 4
    # enough units for no split: 200 sequences x 8 K/V heads x 1 tile = 1600
    assert lib.paged_attn_multi_query_workspace_size(200, 32, 8, 8, D, B, MB, 0) == 16 + 200 * 8


# Each case has one defect that the host checks catch before any CUDA call, so no
# pointer is ever used; "big" sizes need more than the 32 MiB scratch array.
_SMALL = dict(S=4, H=2, D=64, B=16, MB=4, NB=16, dt=1, scale=0.125, pt=0, q=0x10000, out=0x10000)
_BIG = dict(_SMALL, S=64, H=64, D=128, MB=2048, pt=16)
_CASES = {
    "bad dtype, big sizes": (dict(_BIG, dt=7), PKV_EDTYPE),
    "bad dtype, no sequences": (dict(_SMALL, S=0, dt=7), PKV_EDTYPE),
    "no sequences": (dict(_SMALL, S=0), PKV_OK),
    "no sequences, big sizes": (dict(_BIG, S=0), PKV_OK),
    "no heads": (dict(_SMALL, H=0), PKV_EINVAL),
    "head_dim 80": (dict(_SMALL, D=80), PKV_EUNSUPPORTED),
    "block size 24": (dict(_SMALL, B=24), PKV_EUNSUPPORTED),
    "partition not a multiple of B": (dict(_SMALL, pt=17), PKV_EINVAL),
    "no blocks, big sizes": (dict(_BIG, NB=0), PKV_EINVAL),
    "nan scale, big sizes": (dict(_BIG, scale=float("nan")), PKV_EINVAL),
    "null q, big sizes": (dict(_BIG, q=0), PKV_EINVAL),
    "misaligned out, big sizes": (dict(_BIG, out=0x10004), PKV_EALIGN),
    "big sizes": (_BIG, PKV_EWORKSPACE),
}


@pytest.mark.parametrize("name", sorted(_CASES))
def test_noalloc_returns_what_decode_returns(lib, name):
    """The allocation-free decode runs the argument checks of paged_attn_decode in
    the same order, with its scratch array standing in for a workspace of
    PKV_NOALLOC_SCRATCH_BYTES: both return the same code for the same arguments."""
    a, want = _CASES[name]
    fake = 0x10000
    common = (a["q"], fake, fake, fake, fake, a["S"], a["H"], a["D"], a["B"], a["MB"], a["NB"], a["dt"],
              ctypes.c_float(a["scale"]), a["out"], a["pt"])
    got_noalloc = lib.paged_attn_decode_noalloc(*common, None)
    got_decode = lib.paged_attn_decode(*common, 0x20000, _lib.NOALLOC_SCRATCH_BYTES, None)
    assert got_decode == want, (name, got_decode)
    assert got_noalloc == want, (name, got_noalloc)


PKV_EOVERLAP = -11


@pytest.mark.parametrize("pairs,want", [
    ([], PKV_OK),
    ([[3, 9]], PKV_OK),
    ([[3, 9], [3, 10], [3, 11]], PKV_OK),            # one shared block forked three times
    ([[3, 9], [4, 10]], PKV_OK),
    ([[3, 3]], PKV_EOVERLAP),                        # src == dst
    ([[3, 9], [4, 9]], PKV_EOVERLAP),                # a dst repeats
    ([[3, 9], [9, 10]], PKV_EOVERLAP),               # a dst is also a src (chained copy)
    ([[9, 10], [3, 9]], PKV_EOVERLAP),               # ... in either order
    ([[-1, 5], [7, -1]], PKV_OK),                    # out-of-range ids are the device's to flag
])
def test_check_copy_pairs(lib, pairs, want):
    import paged_kv_cache_328_b200 as pkv
    assert pkv.check_copy_pairs(pairs) == want


@pytest.mark.parametrize("slots,want", [
    ([], PKV_OK), ([5, 6, 7], PKV_OK), ([-1, -1, 4], PKV_OK), ([5, 6, 5], PKV_EOVERLAP), ([0, 0], PKV_EOVERLAP),
])
def test_check_slots(lib, slots, want):
    import paged_kv_cache_328_b200 as pkv
    assert pkv.check_slots(slots) == want


def test_check_argument_errors_and_toggle(lib):
    assert lib.pkv_check_copy_pairs(None, 1) == PKV_EINVAL
    assert lib.pkv_check_slots(None, -1) == PKV_EINVAL
    import paged_kv_cache_328_b200 as pkv
    before = pkv.set_debug_checks(None)
    assert pkv.set_debug_checks(True) == before
    assert pkv.set_debug_checks(None) is True
    assert pkv.set_debug_checks(False) is True
    assert pkv.set_debug_checks(None) is False
    pkv.set_debug_checks(before)
    assert _lib.strerror(PKV_EOVERLAP) != "unknown error code"


def test_debug_checks_follow_the_environment():
    """PKV_CHECK=1 turns the checks on at the first query (a fresh process)."""
    import subprocess
    import sys
    code = ("import paged_kv_cache_328_b200 as p; import sys; "
            "sys.exit(0 if p.set_debug_checks(None) else 3)")
    env = dict(os.environ, PKV_CHECK="1")
    assert subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env).returncode == 0
    env["PKV_CHECK"] = "0"
    assert subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env).returncode == 3
