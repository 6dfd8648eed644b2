"""DSA (DeepSeek Sparse Attention) decode path for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libdsa_b200.so`` built from ``csrc/``;
``dsa`` is its thin Python binding (argument marshalling only).
"""
