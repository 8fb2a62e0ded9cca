"""Plain fp64 CPU oracle of the hybrid CSA/HCA decode path.

TEST INFRASTRUCTURE.  Only the test suite, the package entry's smoke check and
the benchmark's CPU-baseline / reference arm may import this package.  The
CUDA library never calls it and shares no code with it.

Everything here is written from the method as the following web pages state
it (cited by page and section in each function):

  [SW] shareware.cn/news/167317 -- essay on DeepSeek V4 Hybrid Attention
       (CSA, HCA, Lightning Indexer, sliding window, MQA, attention sink);
       sections numbered in Chinese: §二 ... §十四.
  [TR] trdm.cn/news/516303 -- "从 MLA 到 CSA，聊聊大模型 Attention 的瘦身与闪送"
       (prior art MHA/MQA/GQA/MLA, FlashAttention, PagedAttention, NSA/DSA,
       and V4's CSA/HCA in §4.3).
  [AM] aimodeling.com news "DeepSeek V4 混合注意力架构解析：如何在1M上下文下将
       计算量降至原来的27%？" (ratios 4:1 / 128:1, top-1024, 128-token window).

All arithmetic is float64 on values decoded exactly from their storage form
(bf16, fp32, OCP E4M3).  Where floating point decides an integer -- the E4M3 codes
of pooled indexer keys and of FP8 main-KV rows -- the definition is exact
(indexer.pool_keys_f64, quantize_keys_f64; kv8.quantize_rows_f64) and
indexer.quotient_error_bound / kv8.quotient_error_bound say where an fp32 evaluation
may round to the neighbouring code; indexer.pool_keys / quantize_keys restate the
same steps in fp32 (the kernel's precision) as a second, labelled check.
Loops are vectorised with numpy but follow each definition term by term; nothing
is blocked, fused or reordered beyond it.

Parity status of each function is stated in its docstring; every function
here is pinned by the ``-m "not gpu"`` tests in ``tests/test_oracle_*.py``.
"""

from . import codecs, compress, indexer, attention, norm, step  # noqa: F401
