"""B200-native GQA attention over a static, sequence-major KV cache.

The compute lives in ``libarkattn.so`` (hand-written CUDA for sm_100a behind a
plain C ABI, declared in ``include/arkattn.h``).  ``gqa_attention_static_b200.ops``
is a thin ctypes binding with the same entry-point names; ``workloads`` builds
seeded synthetic inputs.
"""
