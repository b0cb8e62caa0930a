"""BitLinear W1.58A8 forward on B200 (sm_100a).

Ternary weights {-1, 0, +1} with one absmean scale per matrix, int8
activations quantised per token by absmax, int32 accumulation and a fused
rescale, as hand-written CUDA behind the C ABI of ``include/bitlinear.h``;
and the 1-bit variant with weights Sign(W - mean(W)) in {-1, +1}.
"""
from .bitlinear import (ENGINES, BatchPlan, BitLinear, BitLinearError, DecoderBlock, binarize_weights,
                        decode_engine, device_status, forward, forward_acc, forward_binary,
                        forward_binary_acc, forward_binary_fp, forward_fp, forward_fp_batch,
                        forward_fp_workspace, forward_noalloc, forward_workspace, get_decode_engine,
                        glu_forward, lib, num_sms, pack, pack_bits, quant_act, quant_act_rms,
                        quantize_weights, set_decode_engine, status_string)

__all__ = ["ENGINES", "BatchPlan", "BitLinear", "BitLinearError", "DecoderBlock", "binarize_weights",
           "decode_engine", "device_status", "forward", "forward_acc", "forward_binary", "forward_binary_acc",
           "forward_binary_fp", "forward_fp", "forward_fp_batch", "forward_fp_workspace", "forward_noalloc",
           "forward_workspace", "get_decode_engine", "glu_forward", "lib", "num_sms", "pack", "pack_bits",
           "quant_act", "quant_act_rms", "quantize_weights", "set_decode_engine", "status_string"]
