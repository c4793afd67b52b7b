"""CPU oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import, call or link anything here. The product path
(the CUDA library and its binding) never does, and the two share no code: the
oracle restates the definitions on the pages in plain fp64 code.

Pages cited (by title and section):
  [KV-04] "04. 注意力与 KV 缓存" (inference series, niuwancheng.cn)
  [HB-07] "07｜KV Cache、FlashAttention与PagedAttention的内部过程"
          (AI engineering handbook, chapter 07; questions Q025-Q028)
  [CN-06] "06 KV Cache、Prefix Cache、PagedAttention 与 vLLM"
          (course notes, sections 6.1-6.7)
  [KV-03] "03. KV Cache：用显存换计算" (llm-inference series, niuwancheng.cn)

Modules:
  reference   attention definitions, online-softmax merge, slot and block
              arithmetic, KV-bytes formula, fp64 paged decode (C, OpenMP)
  pool_model  refcounted FIFO page pool and brute-force prefix index
  rope        rotary position embedding of q / k ahead of the KV append
              ([CN-06] 6.1), exact and at stored precision
  fp8         E4M3 K/V cache: format, quantising append, fp64 decode over
              the read values
"""
from . import reference, pool_model, rope, fp8  # noqa: F401
