"""Sparse ternary BitLinear (Sparse-BitNet hot path) for NVIDIA B200 (sm_100a).

The compute lives in libbitnet_sparse.so (CUDA kernels behind a C ABI, see
include/bitnet_sparse.h); this package is its thin Python binding plus the
seeded synthetic input generators.
"""
from ._abi import (  # noqa: F401
    BITNET_BF16, BITNET_F32, BitnetChainOp, BitnetError, BitnetPackedW, BitnetPackItem, DecodeChain, PackBatch, PackedWeights, Workspace,
    bitnet_decode_chain, bitnet_dgrad, bitnet_pack_nm_update_batch, bitnet_pack_6of8_windows,
    bitnet_quant_act_lift_6of8, packed_6of8, bitnet_pack_nm, bitnet_pack_nm_update, bitnet_quant_act, bitnet_rmsnorm_quant, bitnet_swiglu_quant, bitnet_wgrad, bitnet_adamw_step, AdamWBatch, adam_bias_correction, bitnet_quant_linear, bitnet_read_device_status, bitnet_wait_selftest, bitnet_tensor_peak, bitnet_sparse_linear, load,
)

__all__ = [
    "PackedWeights", "Workspace", "BitnetError", "BitnetPackedW", "BitnetChainOp", "DecodeChain", "load",
    "bitnet_decode_chain", "bitnet_pack_nm_update_batch", "PackBatch", "BitnetPackItem",
    "bitnet_pack_6of8_windows", "bitnet_quant_act_lift_6of8", "packed_6of8",
    "bitnet_pack_nm", "bitnet_pack_nm_update", "bitnet_quant_act", "bitnet_rmsnorm_quant", "bitnet_swiglu_quant", "bitnet_wgrad", "bitnet_adamw_step", "AdamWBatch", "adam_bias_correction", "bitnet_quant_linear", "bitnet_sparse_linear", "bitnet_dgrad", "bitnet_read_device_status", "bitnet_wait_selftest", "bitnet_tensor_peak",
    "BITNET_F32", "BITNET_BF16",
]
