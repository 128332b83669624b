"""Slim attention (K-only context cache) decode hot path for B200 (sm_100a).

The compute path is the native library ``libslim.so`` built from ``csrc/``;
``only_cache_exact_b200.slim`` is its ctypes binding. Importing this package
does not load the library, so the CPU-only parts (``synth``, ``params``) work
on machines without a GPU; ``replicas`` holds the host logic of the
one-process-per-GPU runs.
"""

__all__ = ["slim", "synth", "params", "replicas"]
