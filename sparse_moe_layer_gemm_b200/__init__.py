"""B200-native (sm_100a) forward of the Step-3.5-Flash sparse-MoE FFN layer.

The layer runs in the C-ABI library ``libmoe.so`` (declared in
``include/moe.h``); :mod:`sparse_moe_layer_gemm_b200.binding` marshals torch
tensors into it.  Importing this package loads no native code; the first call
that needs the library loads it and raises if it is missing.
"""
__all__ = ["binding", "workloads", "roofline"]
