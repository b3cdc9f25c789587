"""CPU oracle for the paged decode path -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously correct NumPy (fp64 for floating point) restatements of
what the path computes, written from three web pages on PagedAttention:

  * "What is PagedAttention? Definition & Virtual Memory Architecture in
    Enterprise AI" (esaholic.com AI glossary) -- called *Glossary* below;
  * "Paged Attention" (invest-in.ai AI terminology) -- *Terminology*;
  * "PagedAttention Internals: How Memory Fragmentation in LLM Serving Was
    Solved" (dailyaiworld.com) -- *Internals*.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import anything here.  Nothing in this package imports the
CUDA path or its Python binding, and the CUDA path never imports this package.

Modules
  allocator  ref-counted free-page pool, block tables, fork, copy-on-write
  cache_ops  writing tokens into page slots; whole-page copies
  attention  block-table gather + textbook softmax attention (fp64); the
             split-context partials and their log-sum-exp merge; several
             causal query tokens per sequence (draft verification)
  formulas   block counts, KV bytes per token, internal waste
  scenario   runs a workload trace through the pieces above

Every function is pinned by ``tests/test_oracle_*.py`` against facts the pages
print, closed forms, a library routine, or brute force; none is "parity
unpinned".
"""
