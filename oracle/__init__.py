"""CPU oracle for paged decode attention and its two cache-maintenance operations.

This package is TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline / reference arm of ``bench.py`` may import it.  It shares no
code, constant, header or helper with the CUDA library in ``paged_kv_cache_328_b200``
and imports nothing from it; both sides receive the same seeded inputs and
nothing else.  The product path never calls into this package.

Everything is plain NumPy in float64 (the pages fix no precision), written to be
checked against the pages by eye:

* ``storage``          exact widening of stored fp32 / fp16 / bf16 elements to float64.
* ``paged_attention``  gather a sequence's K/V through its block table into a
                       contiguous array, then softmax(scale * K q) V.
* ``cache_ops``        per-token append into slots, copy-on-write block copy,
                       block swaps to and from host memory, and the plain
                       gather used to check indexing.
* ``block_manager``    the host bookkeeping: free list, reference counts,
                       on-demand blocks, copy-on-write trigger, swap lists.

Sources (cited by page title and section):

* [digest]  "PagedAttention - Efficient Memory Management for LLM Serving with vLLM"
            (irregular6612.github.io paper digest): section "Method (PagedAttention +
            vLLM)", the framework-overview flowchart under "방법 (Method)", the
            glossary "핵심 용어 정리".
* [blog]    "vLLM PagedAttention and continuous-batching architecture"
            (tech.blogsailing.com): section 2 "vLLM PagedAttention의 핵심 아키텍처 원리".
* [velog]   "LLM Inference 8 - PagedAttention" (velog.io): sections "KV Cache의 메모리
            문제", "PagedAttention", "PagedAttention의 동작 방식".
* [video]   "KV 캐시·PagedAttention로 LLM 추론 속도와 GPU 처리량 높이기" (allinfo.ai.kr):
            section "쉽게 이해하기".

Parity status: every public function here is pinned by ``tests/test_oracle_pins.py``
(brute force, library routines, closed forms, invariants and the pages' worked
block tables under ``tests/golden/``); none is "parity unpinned".
"""

from .storage import to_f64, STORAGE_DTYPES
from .paged_attention import (
    gather_rows,
    attend,
    softmax_weights,
    paged_decode,
    paged_decode_selected,
    paged_multi_query,
)
from .cache_ops import kv_append, kv_block_copy, gather_kv, kv_swap_out, kv_swap_in
from .block_manager import BlockManager, BlockManagerError

__all__ = [
    "to_f64",
    "STORAGE_DTYPES",
    "gather_rows",
    "attend",
    "softmax_weights",
    "paged_decode",
    "paged_decode_selected",
    "paged_multi_query",
    "kv_append",
    "kv_block_copy",
    "gather_kv",
    "kv_swap_out",
    "kv_swap_in",
    "BlockManager",
    "BlockManagerError",
]
