"""BinaryAttention forward pass for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libbinattn.so`` (hand-written CUDA);
``diffusion_transformers_b200.binattn`` is its thin ctypes binding. This
``__init__`` imports nothing heavy so that the input generator can be used
without the GPU library.
"""
