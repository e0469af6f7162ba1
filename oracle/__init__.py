"""fp64 CPU oracle for grouped-query attention (MHA / GQA / MQA / absorbed MLA).

This package is TEST INFRASTRUCTURE.  Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline / reference legs of ``bench.py`` may
import it.  The product path (the CUDA library and its Python binding) never
imports, links or executes anything here, and this package never imports the
product: the two share no code.  The only thing both sides use is the seeded
input generator module (``attention_mqa_gqa_b200.workloads``), which holds no
attention arithmetic.

Contents
--------
``attention``  numpy fp64 implementation of the definition (tests, small and
               sampled cases).
``c_oracle``   ctypes front of ``attn_oracle.c``, the same definition written
               again in plain C with pthreads (large cases, CPU timing).
"""
