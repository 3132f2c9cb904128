"""B200-native OrbitQuant online quantized-linear path.

RPBH rotation -> per-token norm -> Lloyd-Max nearest-centroid codes (``oq_quantize_act``),
and a codebook GEMM against pre-quantized weights scaled by s * row_norm (``oq_linear``),
carried by hand-written sm_100a CUDA kernels behind the C ABI in ``include/oq.h``.

``calibration_free_bit_b200.oq`` is the thin Python binding (argument marshalling only);
``calibration_free_bit_b200.synth`` holds the seeded synthetic workloads.
"""
__all__ = ["oq", "synth"]
