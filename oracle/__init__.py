"""CPU oracle for paged-KV attention: TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, fp64 statement of what the attention path
computes.  It exists so that tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` can check and time
the CUDA library against an independent definition.  Nothing in the product
package imports it, and it imports nothing from the product package: the two
share no code, constants or helpers.  Inputs reach it as NumPy arrays produced
by the seeded workload generators.

Modules
-------
codecs     bit-level bfloat16 and OCP FP8 E4M3 codecs
attention  slot gather, decode, extend, LSE merge, materialised N x N reference
sage       8-bit Sage decode following the pages' formula step by step
plan       the integer split-KV / tile work-list algorithm

Every function names the passage of the source pages it restates.  The pages
are cited by title and section:

* "Implement Flash Attention Back End in SGLang - Basics and KV Cache"
  (hnr.moe), the KV-cache and forward-mode passages;
* "SGLang의 FA3 디코드 최적화: get_scheduler_metadata 도입", sections
  "코드 분석" (code analysis) and "왜 이게 좋은가" (why it helps);
* "FlashInfer PrimTS, Sage Attention 도입으로 8비트 양자화 및 성능 최적화 달성",
  section "코드 분석" items 1 (README "Sage attention") and 4 (kernel-level
  scale application);
* "FlashAttention: 优化计算过程中的临时显存占用" sections 1-2, and
  "PagedAttention: 优化 KV Cache 的管理和利用率" section 2 (工作原理);
* "Flash Attention Backend in SGLang: Grundlagen und KV Cache optimal nutzen".

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, library routines, brute force or the pages' printed
figures; none is "parity unpinned".
"""
