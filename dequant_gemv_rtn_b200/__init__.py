"""dequant_gemv_rtn_b200: RTN group-wise 4-bit weight quantization (INT4 asymmetric,
FP4 E2M1, AFPQ, RaZeR; INT8 / FP16 for selectively raised modules) and the
decode-time fused-dequant GEMV / small-batch GEMM, as hand-written CUDA for
NVIDIA B200 (sm_100a) behind a C ABI (include/qnt.h, libqnt.so).

The C-ABI binding lives in ``dequant_gemv_rtn_b200.qnt`` (loading it requires
the built libqnt.so); ``dequant_gemv_rtn_b200.synth`` draws seeded inputs.
"""
__all__ = ["qnt", "synth", "build"]
