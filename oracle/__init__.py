"""Float64 CPU oracle for paged-attention decode. TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may import this package. The product (the C-ABI library and its
Python binding) never calls it and has no CPU fallback through it.

It is plain, slow and written to be checked by eye against its sources:

* vLLM pages, "PagedAttention" (dingiv.github.io/ai/compute/engine/vllm):
  KV cache cut into fixed 16-token pages scattered through memory; a position's
  page is ``position // block_size``; a Block Manager hands out and takes back
  pages in O(1) with a free list.
* "vLLM 前世今生" section 3.2 (hncyxsy.com/news/276126): default block of 16 tokens,
  physical blocks need not be contiguous, a block table maps them, several
  sequences may point at one physical block (prefix sharing).
* The decode operation itself is softmax(scale * q K^T) V over the whole context
  of the sequence, computed here as that definition in float64, max-subtracted,
  with no online form, no partitions and no blocking.
* The FP8 codec follows the OCP 8-bit floating point specification (E4M3:
  bias 7, no infinities, S.1111.111 is NaN, largest finite 448).

Modules: ``paging`` (page index, slots, free-list model, block tables),
``e4m3`` (FP8 codec), ``cache`` (reshape_and_cache scatter), ``attention``
(decode). It shares no code with ``paged_kv_cache_385_b200``; both consume the
seeded inputs of ``workloads``.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, brute force, library routines or the pages' worked
example; none is "parity unpinned".
"""
from . import attention, cache, e4m3, paging  # noqa: F401
