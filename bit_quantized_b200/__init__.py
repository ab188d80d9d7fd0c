"""B200 (sm_100a) 8-bit quantized linear layer.

``bit_quantized_b200.q8`` is the Python binding of ``libq8.so`` (include/q8.h);
``bit_quantized_b200.build`` compiles that library in-tree with nvcc.
"""
__all__ = ["q8", "build"]
