"""CPU oracle for paged KV-cache decode — TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct fp64 restatements of what the paged decode path
computes, used to check the CUDA library.  Only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs may
import this package.  It shares no code with ``paged_kv_cache_406_b200`` and
imports nothing from it; inputs reach it as plain numpy arrays.

Sources (cited by page title and section):

* "vLLM's 'memory paging' — PagedAttention illustrated" (vLLM的'内存分页'到底多神奇),
  §2 (pages, per-sequence page table, free page list) and §3 (phase 1:
  allocation / page-table growth; phase 2: gather pages and run standard
  attention; phase 3: reclaim, shared prefix pages with reference counts),
  §4 (admission control, abort).
* "LLM inference optimisation: principles overview" (LLM 推理优化：技术原理解析总览),
  §2.2 domain three and §3.3 (KV cache cut into fixed-size physical pages of
  16 tokens, logical-to-physical page table, O(1) append), §2.3 (chunked
  prefill of long inputs).
* the vLLM production-deployment page, §2 (chunked prefill and decode steps
  batched together; prefix blocks shared between requests) and §5 (prefix
  caching).

Modules:

* :mod:`oracle.paged_attention` — gather through the block table, two-pass fp64
  softmax attention with GQA head grouping, KV append by slot mapping, block
  copy, the split-partition (m, l, o) rescaling identity, and causal chunked
  prefill attention over the pool (each new row sees its own prefix).
* :mod:`oracle.block_allocator` — a pure-Python model of the host block
  allocator (free stack, refcounts, copy-on-write, all-or-nothing errors).
* :mod:`oracle.fp8` — e4m3 codes (decode, round-to-nearest-even saturating
  encode), the quantising append and decode attention over e4m3 pools with
  per-pool scales ("LLM inference optimisation: principles overview" §5.1:
  an FP8 KV cache).

Parity status: every function here is pinned by ``tests/test_oracle.py``,
``tests/test_oracle_prefill.py``, ``tests/test_oracle_fp8.py`` or
``tests/test_allocator_oracle.py`` against something other than itself
(brute force, a library special case, closed forms, invariants, the worked
paging example of the vLLM paging page; for e4m3, torch's float8_e4m3fn and
closed-form code values); none is "parity unpinned".
"""
