"""invariant_bi_lora_b200: deterministic-reduction kernels for NVIDIA B200 (sm_100a).

The compute lives in ``libbi.so`` (hand-written CUDA behind a C ABI declared in
``include/bi.h``).  ``invariant_bi_lora_b200.bi`` is the thin ctypes binding
with the same names; it loads the library on first use and raises if it is
missing.  ``invariant_bi_lora_b200.synth`` draws the seeded synthetic inputs.
"""

__all__ = ["bi", "synth"]
