"""Expert-routed MoE FFN layer for NVIDIA B200 (sm_100a).

The layer (route -> expert-major plan -> grouped SwiGLU experts over W4/W8/BF16
weights -> fixed-order weighted combine) runs in the CUDA library built from
``csrc/`` and declared in ``include/moe_b200.h``; ``binding`` is its Python
front end, ``synth`` the seeded input generator.
"""
__all__ = ["binding", "synth"]
