"""CPU oracle for paged-KV attention.  TEST INFRASTRUCTURE, NOT PRODUCT CODE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of
``bench.py`` (including ``bench.py --impl reference``) may import this
package.  The CUDA library never calls it and has no CPU fallback to it.

It is a plain, slow, obviously-correct restatement, in float64 NumPy, of
what the pages define:

* ``block_manager`` -- the block manager of the page "LLM 推理引擎
  Continuous Batching 与 PagedAttention" (§3.2 核心数据结构), with the
  refcounted shared prefix of §4.1 (KV Cache 的 Shared Prefix).
* ``attention`` -- paged attention as the page's §3.3 (GPU Kernel 中的分页读取)
  states it: each sequence's K/V is read through its block table
  (physical block = table[pos // block_size], row pos % block_size), then
  softmax(q K^T * scale) V per head, in float64 with max subtraction; the
  chunked prefill of §4.3 is the same computation restricted causally.
* ``sizes`` -- the KV-bytes-per-token closed form of §1.2 and the block
  count / internal-waste arithmetic of §3.2 and §3.4.
* ``workloads`` -- replays the seeded workload recipes (``synth_inputs``)
  through the oracle block manager and builds the cache the step reads.

Every function is pinned by the ``-m "not gpu"`` tests against facts the
pages and mathematics fix (closed forms, ``torch``'s scaled-dot-product
attention on CPU, permutation invariance, special cases, brute force).
No part of this package is "parity unpinned".
"""
