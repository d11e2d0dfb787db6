"""Reference oracle for the paged KV-cache decode path — test infrastructure only.

A plain, slow CPU restatement of what the path computes, in float64 for the
attention arithmetic and in exact integer/bit operations for the cache writes,
block copies and block-manager bookkeeping. It exists to check the CUDA path,
not to serve it: only the test suite, the package smoke check and the CPU-baseline
leg of the benchmark may import it. It shares no code with the CUDA library
(kernels, headers, helpers, constants) and does not import it; the only module
both sides use is ``workloads``, which draws the seeded inputs.

Sources are the three pages on the subject:
  * "PagedAttention and Continuous Batching" (roadtointelligence.com) — sections
    "Pages, from operating systems" (block table, on-demand blocks, the 70-token
    worked example, copy-on-write sharing) and "Batch by step, not by request";
  * "vLLM: PagedAttention and continuous batching" (llmstudy.shddai.net) — the
    direct answer (attention follows the block-table mapping);
  * "PagedAttention: The vLLM Paper" (ai.zenoagi.com) — "The Core Idea" (block
    pool and block-table figure), "The OS paging analogy", "Implementation
    Essentials" (block manager with pool, reclamation and refcounts).

Modules:
  fpbits         exact decode of fp16 / bf16 bit patterns to float64
  block_manager  pool, block tables, slot mapping, refcounts, copy-on-write
  cache_ops      writing new tokens into their slots; whole-block copies
  attention      gather through the block table + naive softmax(q K^T * scale) V,
                 and the split-KV partial state with its log-sum-exp merge
  step           one decode step of a workload, end to end, on the oracle side

Parity status: every function here is pinned by tests/test_oracle_pins.py
against the pages' worked example and figure, closed forms, invariants,
brute force on tiny inputs and a library attention routine; none is unpinned.
"""
