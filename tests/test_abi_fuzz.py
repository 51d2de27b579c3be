"""Property tests of the pure host queries of the C ABI (no GPU): for any integers,
the workspace and partition queries return without crashing, reject exactly the
same argument sets, and accepted sizes follow the documented workspace layout."""

import ctypes

import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

from paged_kv_cache_328_b200 import _lib  # noqa: E402
from paged_kv_cache_328_b200 import build as builder  # noqa: E402

BAD = ctypes.c_size_t(-1).value
ints = st.one_of(st.integers(-3, 300), st.sampled_from([0, 1, 64, 128, 4096, 65535, 65536, 1 << 20, 2 ** 31 - 1]))


@pytest.fixture(scope="module")
def lib():
    builder.build()
    return _lib.load()


def round16(n):
    return (n + 15) // 16 * 16


@settings(max_examples=400, deadline=None)
@given(S=ints, H=ints, D=st.sampled_from([32, 64, 96, 128, 256, -1]), B=st.sampled_from([4, 8, 16, 24, 32, 64, 128, 256, 0]),
       MB=ints, pt=ints)
def test_decode_queries_agree(lib, S, H, D, B, MB, pt):
    n = lib.paged_attn_decode_workspace_size(S, H, D, B, MB, pt)
    p = lib.paged_attn_decode_partition_tokens(S, H, D, B, MB, pt)
    assert (n == BAD) == (p < 0)
    if n != BAD:
        max_ctx = MB * B
        assert 0 < p <= max_ctx and p % B == 0
        parts = -(-max_ctx // p)
        expect = 16 + round16(S * parts * 8)
        if parts > 1:
            expect += round16(S * H * parts * 8) + round16(S * H * parts * D * 4)
        assert n == expect


@settings(max_examples=300, deadline=None)
@given(S=ints, H=ints, Hkv=st.sampled_from([1, 2, 3, 8, 0, -1]), D=st.sampled_from([64, 128, 80]),
       B=st.sampled_from([8, 16, 128]), MB=ints, pt=ints, Lq=st.sampled_from([1, 2, 17, 64, 0]))
def test_grouped_and_multi_token_queries_never_crash(lib, S, H, Hkv, D, B, MB, pt, Lq):
    g = lib.paged_attn_decode_gqa_workspace_size(S, H, Hkv, D, B, MB, pt)
    gp = lib.paged_attn_decode_gqa_partition_tokens(S, H, Hkv, D, B, MB, pt)
    assert (g == BAD) == (gp < 0)
    m = lib.paged_attn_multi_query_workspace_size(S, Lq, H, Hkv, D, B, MB, pt)
    if Lq <= 0 or Hkv <= 0 or H <= 0 or H % Hkv:
        assert m == BAD
    # the tuner's workspace covers every candidate it times, the library's own choice among them
    t = lib.paged_attn_decode_tune_workspace_size(S, H, Hkv, D, B, MB)
    g0 = lib.paged_attn_decode_gqa_workspace_size(S, H, Hkv, D, B, MB, 0)
    if t != BAD and g0 != BAD:
        assert t >= g0
