"""HQQ group-wise weight quantization on B200 (sm_100a).

The CUDA library is loaded by the submodule ``free_weight_quantization_b200.hqq``; importing
this package alone loads nothing.
"""
