"""Plain, slow CPU oracle of the Fast-dLLM block-wise DualCache decoder.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code with
the CUDA library (``kv_cache_decode_dualcache_b200``) and imports nothing from
it; both sides receive the same inputs (weights, prompts) from the seeded input
generator, which holds none of the method's arithmetic.

Sources followed (page title, then section):

* "Fast-dLLM：NVIDIA研究团队通过KV缓存和并行解码实现扩散大语言模型的无训练加速"
  (techwalker.com, 2025-06-03), section "核心创新：适合扩散模型的KV缓存"
  (block procedure: compute and keep the other blocks' KV before a block,
  recompute all KV after it; DualCache keeps prefix and suffix) and section
  "解决并行解码的质量下降问题" (threshold on per-token confidence instead of a
  fixed count).
* Fast-dLLM overview on ccyt168.com, section 一 "核心技术", item 1
  "分块 KV 缓存" (DualCache caches the prompt prefix and the masked suffix) and
  item 2 "置信度感知并行解码" (confidence = the probability the model gives the
  token; threshold e.g. 0.9; the (n+1)·eps <= 1 parallel = sequential result).

Modules:

* ``numerics``  - bf16 round-to-nearest-even emulation, SiLU, log-sum-exp.
* ``model``     - the bidirectional transformer ``f`` (RMSNorm, RoPE, attention
                  without a mask, SwiGLU, scaled LM head) in float64, with
                  explicit per-position K/V so cached and fresh K/V meet in one
                  attention routine.
* ``decode``    - confidence / argmax, the threshold-or-fallback unmask rule,
                  block-wise generation in cache modes none / prefix / dual, and
                  the teacher-forced single step.
* ``theorem``   - a toy "model" built from an explicit joint table, used to
                  check the (n+1)·eps <= 1 statement by brute force.
* ``similarity``- cosine similarity of two steps' K/V activations per layer
                  and position (the diagnostic behind the approximate cache).

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, independent library routines (torch CPU float64),
invariants the pages fix, or brute force.  What stays unpinned: agreement
with the real Fast-dLLM outputs on trained LLaDA / Dream weights (no weights
and no printed worked example exist), i.e. "parity unpinned" for that claim.
"""
