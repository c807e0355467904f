"""B200-native QLoRA frozen-NF4 linear layer (sm_100a).

The compute path is the C-ABI library ``libqlora_nf4.so`` built from
``csrc/``; ``api`` is a thin ctypes binding over it.  ``inputs`` draws the
seeded synthetic tensors used by the tests and the benchmark.
"""
