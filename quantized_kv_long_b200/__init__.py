"""B200-native attention over a block-quantized KV cache (Q8_0 keys, Q4_0 values).

The compute path is the C-ABI library ``libkvq.so`` (hand-written CUDA for
sm_100a); :mod:`quantized_kv_long_b200.kvq` is its thin ctypes binding and
:mod:`quantized_kv_long_b200.workload` draws the seeded synthetic inputs.
"""
