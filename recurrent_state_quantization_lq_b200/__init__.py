"""Windowed INT8 recurrent-state decode for gated delta-rule attention on B200.

The compute path is the C-ABI library ``liblq`` (hand-written sm_100a CUDA
kernels); ``recurrent_state_quantization_lq_b200.lq`` is its thin Python
binding and ``inputs`` holds the seeded synthetic workloads.
"""
