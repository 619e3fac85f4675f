"""B200-native (sm_100a) MoE-layer forward pass.

The compute path is ``libmoe.so`` (hand-written CUDA for sm_100a behind the
C ABI in ``include/moe.h``); ``mixture_experts_layer_33_b200.moe`` is its
thin ctypes binding and ``mixture_experts_layer_33_b200.inputs`` draws the
seeded synthetic workloads. Importing this package loads nothing; importing
``.moe`` loads the library and raises if it has not been built.
"""

__version__ = "0.1.0"
