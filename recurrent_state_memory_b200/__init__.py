"""B200-native key-axis-gated delta-rule recurrence (chunk-WY forward + recurrent decode).

The compute lives in the CUDA library ``libgdr.so`` (sources under ``csrc/``,
C-ABI declared in ``include/gdr.h``); ``gdr`` is the thin ctypes binding over it.
Importing this package loads nothing; ``recurrent_state_memory_b200.gdr`` loads
the library and fails loudly if it is missing.
"""
__all__ = ["gdr", "inputs"]
