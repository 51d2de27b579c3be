"""ctypes binding of libpagedkv.so (the C ABI in include/pagedkv.h).

Argument marshalling only: every function checks that the tensors are CUDA,
contiguous and of the expected dtypes, passes their device pointers and the
current torch stream to the C entry point of the same name, and raises
``PagedKVError`` on a non-zero return.  There is no fallback: if the shared
library is missing, or a tensor is not on a CUDA device, the call fails.
"""

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpagedkv.so")

PKV_F32, PKV_F16, PKV_BF16 = 0, 1, 2
DTYPE_CODE = {torch.float32: PKV_F32, torch.float16: PKV_F16, torch.bfloat16: PKV_BF16}

ERRORS = {
    0: "PKV_OK", -1: "PKV_EINVAL", -2: "PKV_EDTYPE", -3: "PKV_EALIGN", -4: "PKV_EUNSUPPORTED",
    -5: "PKV_ECUDA", -6: "PKV_EWORKSPACE", -7: "PKV_EDEVICE", -8: "PKV_ETIMEOUT", -9: "PKV_ENOMEM",
    -10: "PKV_ESEQ", -11: "PKV_EOVERLAP",
}
DEVICE_REASONS = {0: "ok", 1: "block id", 2: "context length", 3: "slot", 4: "copy pair", 5: "wait timeout"}

# Every symbol the header declares, with its ctypes signature.
_c_void_p, _c_int, _c_float, _c_size_t = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "paged_attn_decode": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                   _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                   _c_float, _c_void_p, _c_int, _c_void_p, _c_size_t, _c_void_p]),
    "paged_attn_decode_workspace_size": (_c_size_t, [_c_int] * 6),
    "paged_attn_decode_partition_tokens": (_c_int, [_c_int] * 6),
    "kv_cache_append": (_c_int, [_c_void_p] * 5 + [_c_int] * 6 + [_c_void_p]),
    "kv_block_copy": (_c_int, [_c_void_p] * 3 + [_c_int] * 6 + [_c_void_p]),
    "paged_kv_gather": (_c_int, [_c_void_p, _c_void_p] + [_c_int] * 6 + [_c_void_p, _c_void_p]),
    "pkv_get_device_error": (_c_int, [_c_void_p, ctypes.POINTER(_c_int)]),
    "pkv_strerror": (ctypes.c_char_p, [_c_int]),
    "pkv_abi_version": (_c_int, []),
    "paged_attn_decode_gqa": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                       _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                       _c_float, _c_void_p, _c_int, _c_void_p, _c_size_t, _c_void_p]),
    "paged_attn_decode_gqa_workspace_size": (_c_size_t, [_c_int] * 7),
    "paged_attn_decode_gqa_partition_tokens": (_c_int, [_c_int] * 7),
    "paged_attn_multi_query": (_c_int, [_c_void_p] * 5 + [_c_int] * 9 + [_c_float, _c_void_p, _c_int, _c_void_p,
                                                                     _c_size_t, _c_void_p]),
    "paged_attn_multi_query_workspace_size": (_c_size_t, [_c_int] * 8),
    "paged_attn_decode_tune": (_c_int, [_c_void_p] * 5 + [_c_int] * 8 + [_c_float, _c_void_p, _c_void_p,
                                                                     _c_size_t, _c_int, _c_void_p, _c_void_p,
                                                                     _c_int, ctypes.POINTER(_c_int), _c_void_p]),
    "paged_attn_decode_tune_workspace_size": (_c_size_t, [_c_int] * 6),
    "pkv_selftest_wait_timeout": (_c_int, [ctypes.c_longlong, _c_void_p]),
    "kv_blocks_to_host": (_c_int, [_c_void_p] * 3 + [_c_int] + [_c_void_p] * 2 + [_c_int] * 5 + [_c_void_p]),
    "kv_blocks_from_host": (_c_int, [_c_void_p] * 5 + [_c_int] * 6 + [_c_void_p]),
    "pkv_bm_create": (_c_void_p, [_c_int, _c_int, _c_void_p]),
    "pkv_bm_destroy": (None, [_c_void_p]),
    "pkv_bm_add_sequence": (_c_int, [_c_void_p, ctypes.c_int64, _c_int]),
    "pkv_bm_fork": (_c_int, [_c_void_p, ctypes.c_int64, ctypes.c_int64]),
    "pkv_bm_append_tokens": (_c_int, [_c_void_p, _c_void_p, _c_int, _c_void_p, _c_void_p,
                                      ctypes.POINTER(_c_int)]),
    "pkv_bm_free_sequence": (_c_int, [_c_void_p, ctypes.c_int64]),
    "pkv_bm_block_table": (_c_int, [_c_void_p, ctypes.c_int64, _c_void_p, _c_int,
                                    ctypes.POINTER(ctypes.c_int64)]),
    "pkv_bm_fill_tables": (_c_int, [_c_void_p, _c_void_p, _c_int, _c_void_p, _c_int, _c_void_p]),
    "pkv_bm_num_free": (_c_int, [_c_void_p]),
    "pkv_bm_ref_count": (_c_int, [_c_void_p, _c_int]),
    "pkv_bm_swap_out": (_c_int, [_c_void_p, ctypes.c_int64, _c_void_p, _c_int, ctypes.POINTER(_c_int)]),
    "pkv_bm_swap_in": (_c_int, [_c_void_p, ctypes.c_int64, _c_void_p, _c_int, ctypes.POINTER(_c_int)]),
    "pkv_check_copy_pairs": (_c_int, [_c_void_p, _c_int]),
    "pkv_check_slots": (_c_int, [_c_void_p, _c_int]),
    "pkv_set_debug_checks": (_c_int, [_c_int]),
    "paged_attn_decode_noalloc": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                           _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                           _c_float, _c_void_p, _c_int, _c_void_p]),
}
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024


class PagedKVError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        msg = f"{where}: {ERRORS.get(code, code)} ({strerror(code) if _LIB else code})"
        super().__init__(msg)


_LIB = None


def load(path=LIB_PATH):
    """Load the shared library (once) and declare every entry point's signature."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is not built: run `python -m paged_kv_cache_328_b200.build` "
                "(nvcc, sm_100a). There is no CPU fallback.")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def strerror(code):
    return load().pkv_strerror(code).decode()


def abi_version():
    return load().pkv_abi_version()


def _check(rc, where):
    if rc != 0:
        raise PagedKVError(rc, where)


def _cuda(t, name, dtypes=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device}); there is no CPU path")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    return t.data_ptr()


def _stream(device, stream):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _call(fn, args, device, stream):
    """fn(*args, stream) with `device` current; the device is switched only when it is not
    already the current one (entering a device context costs more than the launch)."""
    if device.index is None or device.index == torch.cuda.current_device():
        return fn(*args, _stream(device, stream))
    with torch.cuda.device(device):
        return fn(*args, _stream(device, stream))


def workspace_size(num_seqs, num_heads, head_dim, block_size, max_blocks, partition_tokens=0):
    n = load().paged_attn_decode_workspace_size(num_seqs, num_heads, head_dim, block_size, max_blocks,
                                                partition_tokens)
    if n == ctypes.c_size_t(-1).value:
        raise PagedKVError(-1, "paged_attn_decode_workspace_size")
    return n


def partition_tokens(num_seqs, num_heads, head_dim, block_size, max_blocks, partition_tokens=0):
    rc = load().paged_attn_decode_partition_tokens(num_seqs, num_heads, head_dim, block_size, max_blocks,
                                                   partition_tokens)
    if rc < 0:
        raise PagedKVError(rc, "paged_attn_decode_partition_tokens")
    return rc


def gqa_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks, partition_tokens=0):
    n = load().paged_attn_decode_gqa_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                    max_blocks, partition_tokens)
    if n == ctypes.c_size_t(-1).value:
        raise PagedKVError(-1, "paged_attn_decode_gqa_workspace_size")
    return n


def gqa_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks, partition_tokens=0):
    rc = load().paged_attn_decode_gqa_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                       max_blocks, partition_tokens)
    if rc < 0:
        raise PagedKVError(rc, "paged_attn_decode_gqa_partition_tokens")
    return rc


def alloc_workspace(q, k_cache, block_tables, partition_tokens=0):
    """A uint8 workspace tensor sized for these inputs, on q's device."""
    S, H, D = q.shape
    Hkv, B = k_cache.shape[1], k_cache.shape[2]
    n = gqa_workspace_size(S, H, Hkv, D, B, block_tables.shape[1], partition_tokens)
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def paged_attn_decode(q, k_cache, v_cache, block_tables, context_lens, scale, out=None,
                      partition_tokens=0, workspace=None, stream=None):
    """out[s, h] = softmax(scale * K q) V over the paged context; returns out (float32 [S, H, D]).

    The caches may hold fewer heads than q (grouped-query attention): with Hkv K/V
    heads, query head h reads K/V head h // (H // Hkv).
    """
    lib = load()
    S, H, D = q.shape
    NB, Hkv, B, Dc = k_cache.shape
    if Dc != D or Hkv <= 0 or H % Hkv or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("q [S,H,D] and caches [NB,Hkv,B,D] disagree (H must be a multiple of Hkv)")
    if q.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise TypeError("q, k_cache and v_cache must share one storage dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S, max_blocks] and context_lens [S]")
    _cuda(q, "q", DTYPE_CODE)
    if out is None:
        out = torch.empty((S, H, D), dtype=torch.float32, device=q.device)
    if out.shape != (S, H, D) or out.dtype != torch.float32:
        raise ValueError("out must be float32 [S, H, D]")
    if workspace is None:
        workspace = alloc_workspace(q, k_cache, block_tables, partition_tokens)
    dt = DTYPE_CODE[k_cache.dtype]
    args = (_cuda(q, "q", DTYPE_CODE), _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"),
            _cuda(block_tables, "block_tables", (torch.int32,)),
            _cuda(context_lens, "context_lens", (torch.int32,)),
            S, H, Hkv, D, B, block_tables.shape[1], NB, dt, float(scale),
            _cuda(out, "out", (torch.float32,)), int(partition_tokens),
            _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size())
    if Hkv == H:
        rc = _call(lib.paged_attn_decode, args[:6] + args[7:], q.device, stream)
    else:
        rc = _call(lib.paged_attn_decode_gqa, args, q.device, stream)
    _check(rc, "paged_attn_decode" if Hkv == H else "paged_attn_decode_gqa")
    return out


def kv_cache_append(k, v, k_cache, v_cache, slot_mapping, stream=None):
    """k_cache[slot // B, :, slot % B] = k[t] (and v) for every t with slot >= 0."""
    lib = load()
    T, H, D = k.shape
    NB, Hc, B, Dc = k_cache.shape
    if (Hc, Dc) != (H, D) or v.shape != k.shape or v_cache.shape != k_cache.shape:
        raise ValueError("k/v [T,H,D] and caches [NB,H,B,D] disagree")
    if slot_mapping.shape != (T,):
        raise ValueError("slot_mapping must be [T]")
    if k.dtype != k_cache.dtype or v.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise TypeError("new rows and caches must share one storage dtype")
    args = (_cuda(k, "k", DTYPE_CODE), _cuda(v, "v", DTYPE_CODE), _cuda(k_cache, "k_cache"),
            _cuda(v_cache, "v_cache"), _cuda(slot_mapping, "slot_mapping", (torch.int64,)),
            T, H, D, B, NB, DTYPE_CODE[k_cache.dtype])
    rc = _call(lib.kv_cache_append, args, k_cache.device, stream)
    _check(rc, "kv_cache_append")


def kv_block_copy(k_cache, v_cache, src_dst_pairs, stream=None):
    """k_cache[dst] = k_cache[src] and v_cache[dst] = v_cache[src] for each (src, dst) pair."""
    lib = load()
    NB, H, B, D = k_cache.shape
    if v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype:
        raise ValueError("k_cache and v_cache disagree")
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [n, 2]")
    args = (_cuda(k_cache, "k_cache", DTYPE_CODE), _cuda(v_cache, "v_cache", DTYPE_CODE),
            _cuda(src_dst_pairs, "src_dst_pairs", (torch.int64,)), src_dst_pairs.shape[0],
            H, D, B, NB, DTYPE_CODE[k_cache.dtype])
    rc = _call(lib.kv_block_copy, args, k_cache.device, stream)
    _check(rc, "kv_block_copy")


def _host_int64(a, name):
    import numpy as np
    a = np.ascontiguousarray(np.asarray(a, dtype=np.int64))
    return a, a.ctypes.data if a.size else None


def check_copy_pairs(pairs):
    """PKV_OK (0) or PKV_EOVERLAP for host (src, dst) pairs [n, 2] (no CUDA call)."""
    a, ptr = _host_int64(pairs, "pairs")
    return load().pkv_check_copy_pairs(ptr, a.size // 2)


def check_slots(slots):
    """PKV_OK (0) or PKV_EOVERLAP for a host slot mapping [T] (no CUDA call)."""
    a, ptr = _host_int64(slots, "slots")
    return load().pkv_check_slots(ptr, a.size)


def set_debug_checks(enable):
    """Turn the overlap checks of kv_block_copy / kv_cache_append on or off (None:
    query); returns the previous setting."""
    return bool(load().pkv_set_debug_checks(-1 if enable is None else (1 if enable else 0)))


def paged_kv_gather(cache, block_table_row, context_len, out=None, stream=None):
    """Contiguous [H, context_len, D] copy of one sequence's rows of one pool."""
    lib = load()
    NB, H, B, D = cache.shape
    _cuda(cache, "cache", DTYPE_CODE)
    if out is None:
        out = torch.empty((H, context_len, D), dtype=cache.dtype, device=cache.device)
    if out.shape != (H, context_len, D) or out.dtype != cache.dtype:
        raise ValueError("out must be [H, context_len, D] in the cache dtype")
    args = (_cuda(cache, "cache", DTYPE_CODE), _cuda(block_table_row, "block_table_row", (torch.int32,)),
            int(context_len), H, D, B, NB, DTYPE_CODE[cache.dtype], _cuda(out, "out"))
    rc = _call(lib.paged_kv_gather, args, cache.device, stream)
    _check(rc, "paged_kv_gather")
    return out


def selftest_wait_timeout(limit_cycles=20_000_000, device=None, stream=None):
    """Run the bounded-wait self-test kernel: True when its deliberately stalled wait ran out
    (the device error word then holds PKV_DEV_WAIT_TIMEOUT; read it with get_device_error)."""
    lib = load()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    rc = _call(lambda st: lib.pkv_selftest_wait_timeout(int(limit_cycles), st), (), dev, stream)
    if rc < 0:
        raise PagedKVError(rc, "pkv_selftest_wait_timeout")
    return rc == 1


def get_device_error(device=None, stream=None):
    """Synchronise the stream, read and clear the device error word: (code, reason)."""
    lib = load()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    reason = ctypes.c_int(0)
    rc = _call(lambda st: lib.pkv_get_device_error(st, ctypes.byref(reason)), (), dev, stream)
    return rc, reason.value


def paged_attn_decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, scale, out=None,
                              partition_tokens=0, stream=None):
    """paged_attn_decode with the library's static scratch instead of a workspace.

    For callers that cannot allocate device memory (a host framework that owns all
    of it, or a loop where an allocation's synchronisation is not acceptable): the C
    entry point allocates nothing.  ``out`` must then be passed in by such callers;
    when it is None this wrapper creates it with torch, as a convenience for tests.
    Calls on one device share the scratch: order them on one stream.
    """
    lib = load()
    S, H, D = q.shape
    NB, Hc, B, Dc = k_cache.shape
    if (Hc, Dc) != (H, D) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("q [S,H,D] and caches [NB,H,B,D] disagree")
    if q.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise TypeError("q, k_cache and v_cache must share one storage dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S, max_blocks] and context_lens [S]")
    _cuda(q, "q", DTYPE_CODE)
    if out is None:
        out = torch.empty((S, H, D), dtype=torch.float32, device=q.device)
    if out.shape != (S, H, D) or out.dtype != torch.float32:
        raise ValueError("out must be float32 [S, H, D]")
    args = (_cuda(q, "q", DTYPE_CODE), _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"),
            _cuda(block_tables, "block_tables", (torch.int32,)),
            _cuda(context_lens, "context_lens", (torch.int32,)),
            S, H, D, B, block_tables.shape[1], NB, DTYPE_CODE[k_cache.dtype], float(scale),
            _cuda(out, "out", (torch.float32,)), int(partition_tokens))
    rc = _call(lib.paged_attn_decode_noalloc, args, q.device, stream)
    _check(rc, "paged_attn_decode_noalloc")
    return out


def paged_attn_multi_query(q, k_cache, v_cache, block_tables, context_lens, scale, out=None,
                           partition_tokens=0, workspace=None, stream=None):
    """Several query tokens per sequence: q [S, Lq, H, D] -> out float32 [S, Lq, H, D].

    The Lq new tokens are the last Lq positions of each context (already appended);
    query token j attends the first ctx - Lq + j + 1 tokens.
    """
    lib = load()
    S, Lq, H, D = q.shape
    NB, Hkv, B, Dc = k_cache.shape
    if Dc != D or H % Hkv or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("q [S,Lq,H,D] and caches [NB,Hkv,B,D] disagree")
    if q.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise TypeError("q, k_cache and v_cache must share one storage dtype")
    _cuda(q, "q", DTYPE_CODE)
    if out is None:
        out = torch.empty((S, Lq, H, D), dtype=torch.float32, device=q.device)
    if workspace is None:
        n = lib.paged_attn_multi_query_workspace_size(S, Lq, H, Hkv, D, B, block_tables.shape[1], partition_tokens)
        if n == ctypes.c_size_t(-1).value:
            raise PagedKVError(-1, "paged_attn_multi_query_workspace_size")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    args = (_cuda(q, "q", DTYPE_CODE), _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"),
            _cuda(block_tables, "block_tables", (torch.int32,)),
            _cuda(context_lens, "context_lens", (torch.int32,)),
            S, Lq, H, Hkv, D, B, block_tables.shape[1], NB, DTYPE_CODE[k_cache.dtype], float(scale),
            _cuda(out, "out", (torch.float32,)), int(partition_tokens),
            _cuda(workspace, "workspace"), workspace.numel() * workspace.element_size())
    rc = _call(lib.paged_attn_multi_query, args, q.device, stream)
    _check(rc, "paged_attn_multi_query")
    return out


def _host_pinned(t, name):
    if not isinstance(t, torch.Tensor) or t.device.type != "cpu" or not t.is_pinned() or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous pinned (page-locked) CPU tensor")
    return t.data_ptr()


def kv_blocks_to_host(k_cache, v_cache, block_ids, host_k, host_v, stream=None):
    """host_k[i] = k_cache[block_ids[i]] (and V) into pinned host tensors [n, H, B, D]."""
    lib = load()
    NB, H, B, D = k_cache.shape
    n = block_ids.numel()
    if tuple(host_k.shape) != (n, H, B, D) or host_v.shape != host_k.shape or host_k.dtype != k_cache.dtype:
        raise ValueError("host buffers must be [n, H, B, D] in the cache dtype")
    args = (_cuda(k_cache, "k_cache", DTYPE_CODE), _cuda(v_cache, "v_cache", DTYPE_CODE),
            _cuda(block_ids, "block_ids", (torch.int64,)), n, _host_pinned(host_k, "host_k"),
            _host_pinned(host_v, "host_v"), H, D, B, NB, DTYPE_CODE[k_cache.dtype])
    rc = _call(lib.kv_blocks_to_host, args, k_cache.device, stream)
    _check(rc, "kv_blocks_to_host")


def kv_blocks_from_host(host_k, host_v, k_cache, v_cache, block_ids, stream=None):
    """k_cache[block_ids[i]] = host_k[i] (and V) from pinned host tensors [n, H, B, D]."""
    lib = load()
    NB, H, B, D = k_cache.shape
    n = block_ids.numel()
    if tuple(host_k.shape) != (n, H, B, D) or host_v.shape != host_k.shape or host_k.dtype != k_cache.dtype:
        raise ValueError("host buffers must be [n, H, B, D] in the cache dtype")
    args = (_host_pinned(host_k, "host_k"), _host_pinned(host_v, "host_v"),
            _cuda(k_cache, "k_cache", DTYPE_CODE), _cuda(v_cache, "v_cache", DTYPE_CODE),
            _cuda(block_ids, "block_ids", (torch.int64,)), n, H, D, B, NB, DTYPE_CODE[k_cache.dtype])
    rc = _call(lib.kv_blocks_from_host, args, k_cache.device, stream)
    _check(rc, "kv_blocks_from_host")


class BlockManager:
    """The library's native block manager (host code; no GPU needed).

    Free list, reference counts and per-sequence block tables of one physical
    block pool; see include/pagedkv.h.  Methods raise PagedKVError on failure
    (a failed call changes nothing).
    """

    def __init__(self, num_blocks, block_size, free_order=None):
        self._lib = load()
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        arr = None
        if free_order is not None:
            arr = (ctypes.c_int32 * num_blocks)(*[int(b) for b in free_order])
        self._h = self._lib.pkv_bm_create(self.num_blocks, self.block_size, arr)
        if not self._h:
            raise PagedKVError(-1, "pkv_bm_create")

    def close(self):
        if getattr(self, "_h", None):
            self._lib.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def _rc(self, rc, where):
        if rc < 0:
            raise PagedKVError(rc, where)
        return rc

    def add_sequence(self, seq, num_tokens):
        self._rc(self._lib.pkv_bm_add_sequence(self._h, int(seq), int(num_tokens)), "pkv_bm_add_sequence")

    def fork(self, parent, child):
        self._rc(self._lib.pkv_bm_fork(self._h, int(parent), int(child)), "pkv_bm_fork")

    def append_tokens(self, seqs):
        """One token for each sequence: (slots, [(src, dst), ...] copy-on-write pairs)."""
        n = len(seqs)
        seq_arr = (ctypes.c_int64 * max(1, n))(*[int(x) for x in seqs])
        slots = (ctypes.c_int64 * max(1, n))()
        pairs = (ctypes.c_int64 * max(2, 2 * n))()
        npairs = ctypes.c_int(0)
        self._rc(self._lib.pkv_bm_append_tokens(self._h, seq_arr, n, slots, pairs, ctypes.byref(npairs)),
                 "pkv_bm_append_tokens")
        return list(slots[:n]), [(pairs[2 * i], pairs[2 * i + 1]) for i in range(npairs.value)]

    def free_sequence(self, seq):
        self._rc(self._lib.pkv_bm_free_sequence(self._h, int(seq)), "pkv_bm_free_sequence")

    def block_table(self, seq, max_blocks=None):
        cap = self.num_blocks if max_blocks is None else int(max_blocks)
        row = (ctypes.c_int32 * max(1, cap))()
        tokens = ctypes.c_int64(0)
        n = self._rc(self._lib.pkv_bm_block_table(self._h, int(seq), row, cap, ctypes.byref(tokens)),
                     "pkv_bm_block_table")
        return list(row[:n]), tokens.value

    def fill_tables(self, seqs, max_blocks):
        """Block tables int32 [n, max_blocks] (-1 padded) and context lengths int32 [n] as CPU tensors."""
        n = len(seqs)
        seq_arr = (ctypes.c_int64 * max(1, n))(*[int(x) for x in seqs])
        tables = torch.empty((n, max_blocks), dtype=torch.int32)
        lens = torch.empty((n,), dtype=torch.int32)
        self._rc(self._lib.pkv_bm_fill_tables(self._h, seq_arr, n, tables.data_ptr(), int(max_blocks),
                                              lens.data_ptr()), "pkv_bm_fill_tables")
        return tables, lens

    def num_free(self):
        return self._rc(self._lib.pkv_bm_num_free(self._h), "pkv_bm_num_free")

    def ref_count(self, block):
        return self._rc(self._lib.pkv_bm_ref_count(self._h, int(block)), "pkv_bm_ref_count")

    def swap_out(self, seq):
        blocks = (ctypes.c_int64 * max(1, self.num_blocks))()
        n = ctypes.c_int(0)
        self._rc(self._lib.pkv_bm_swap_out(self._h, int(seq), blocks, self.num_blocks, ctypes.byref(n)),
                 "pkv_bm_swap_out")
        return list(blocks[:n.value])

    def swap_in(self, seq):
        blocks = (ctypes.c_int64 * max(1, self.num_blocks))()
        n = ctypes.c_int(0)
        self._rc(self._lib.pkv_bm_swap_in(self._h, int(seq), blocks, self.num_blocks, ctypes.byref(n)),
                 "pkv_bm_swap_in")
        return list(blocks[:n.value])


def tune_partition_tokens(q, k_cache, v_cache, block_tables, context_lens, scale, reps=5, out=None, stream=None):
    """Time the candidate partition sizes on these inputs; returns (best, {size: ms per call})."""
    lib = load()
    S, H, D = q.shape
    NB, Hkv, B, Dc = k_cache.shape
    if Dc != D or H % Hkv:
        raise ValueError("q [S,H,D] and caches [NB,Hkv,B,D] disagree")
    MB = block_tables.shape[1]
    n = lib.paged_attn_decode_tune_workspace_size(S, H, Hkv, D, B, MB)
    if n == ctypes.c_size_t(-1).value:
        raise PagedKVError(-1, "paged_attn_decode_tune_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((S, H, D), dtype=torch.float32, device=q.device)
    times = (ctypes.c_float * 8)()
    cands = (ctypes.c_int * 8)()
    nc = ctypes.c_int(0)
    args = (_cuda(q, "q", DTYPE_CODE), _cuda(k_cache, "k_cache"), _cuda(v_cache, "v_cache"),
            _cuda(block_tables, "block_tables", (torch.int32,)), _cuda(context_lens, "context_lens", (torch.int32,)),
            S, H, Hkv, D, B, MB, NB, DTYPE_CODE[k_cache.dtype], float(scale), _cuda(out, "out", (torch.float32,)),
            ws.data_ptr(), n, int(reps), times, cands, 8, ctypes.byref(nc))
    rc = _call(lib.paged_attn_decode_tune, args, q.device, stream)
    if rc < 0:
        raise PagedKVError(rc, "paged_attn_decode_tune")
    return rc, {cands[i]: times[i] for i in range(nc.value)}
