"""Context-extended attention forward for B200 (sm_100a).

Scaled-RoPE frequency schedules, Q/K rotation, blockwise causal attention with
online softmax (tcgen05 tensor cores), ring-ordered KV blocks and LSE merge,
exposed through the C ABI of ``librcx.so``; this package is its thin binding.
"""
