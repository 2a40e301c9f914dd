"""B200-native fused MXFP4 routed-MoE layer (sm_100a CUDA behind a C ABI).

The CUDA library ``libmoe_mx.so`` is loaded on first use by
:mod:`block_scaled_moe_softmax_b200.moe_mx`; importing the package itself
loads nothing, so the input generators in :mod:`.workloads` work without a GPU.
"""
