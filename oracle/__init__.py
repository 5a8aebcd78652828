"""CPU oracle for paged decode attention and its block allocator.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this package; only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it.  It shares no code with the CUDA path: it reads the
same seeded inputs (``workloads``) and nothing else.

It is a plain, slow and obviously correct restatement of what three web pages
on paged KV caches fix:

  [P1] "PagedAttention 与在线推理：KV 分页、共享及调度的联合分析"
       (auturnal.com, guides/paged-attention-serving)
  [P2] "PagedAttention：让 KV cache 按需生长"
       (hs-black.github.io, posts/paged-attention)
  [P3] "内存预算约束下的语言模型服务：注意力、分页与调度"
       (auturnal.com, guides/llm-serving-budgets)

Modules:
  accounting  closed forms: KV bytes per token, allocated slots, tail waste,
              position utilisation, pool capacity, swap time
  allocator   the reference block allocator (free queue, refcounts, COW,
              allocate-or-fail, conservation invariant)
  kvops       slot mapping, token append and block copy on NumPy pools
  attention   dense float64 decode attention over the gathered history, the
              online-softmax recurrence and the merge of partial states

Floating point is binary64 throughout.  bf16 inputs arrive as 16-bit patterns
and are widened exactly.

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
values the pages print, closed forms, special cases and brute force.  One
value the pages print has no input on the pages and stays unpinned: the
witness field ``page_tail_slots = 32`` of P3's executed check (its six-request
example is not on the pages).  No oracle function depends on it.
"""
