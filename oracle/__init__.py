"""Oracle package: TEST INFRASTRUCTURE ONLY.

Plain float64 CPU definitions of what the Slim attention decode path computes
(``slim_oracle``) and a fixed-order fp32 GEMM in C (``fp32_gemm.c``, loaded by
``fp32_gemm``). Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline legs may import anything here; the product path never does.
"""
