"""B200-native FP4 quantized linear layer: Hadamard-rotated NVFP4 / MXFP4
quantizers and tcgen05 block-scaled FP4 GEMMs behind a C ABI (include/qfp4.h).

Import ``fp4_precision_b200.qfp4`` for the binding; importing the package
itself loads nothing.
"""
