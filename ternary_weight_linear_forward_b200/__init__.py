"""BitLinear W1.58A8 forward on B200 (sm_100a).

Ternary weights {-1, 0, +1} with one absmean scale per matrix, int8
activations quantised per token by absmax, int32 accumulation and a fused
rescale, as hand-written CUDA behind the C ABI of ``include/bitlinear.h``;
the 1-bit variant with weights Sign(W - mean(W)) in {-1, +1}; group
quantisation along K; and the MatMul-free GLU channel mixer.
"""
from .bitlinear import (BatchPlan, BitLinear, BitLinearError, DecoderBlock, ENGINES, binarize_weights,
                        decode_engine, device_status, forward, forward_acc, forward_binary,
                        forward_binary_acc, forward_binary_fp, forward_fp, forward_fp_batch,
                        forward_fp_workspace, forward_grouped, forward_grouped_acc, forward_grouped_fp,
                        forward_noalloc, forward_path, forward_workspace, get_decode_engine, glu_forward, lib, num_sms,
                        pack, pack_bits, pack_grouped, quant_act, quant_act_grouped, quant_act_rms,
                        quantize_weights, quantize_weights_grouped, set_decode_engine, status_string)

__all__ = ["BatchPlan", "BitLinear", "BitLinearError", "DecoderBlock", "ENGINES", "binarize_weights",
           "decode_engine", "device_status", "forward", "forward_acc", "forward_binary", "forward_binary_acc",
           "forward_binary_fp", "forward_fp", "forward_fp_batch", "forward_fp_workspace", "forward_grouped",
           "forward_grouped_acc", "forward_grouped_fp", "forward_noalloc", "forward_path", "forward_workspace",
           "get_decode_engine", "glu_forward", "lib", "num_sms", "pack", "pack_bits", "pack_grouped",
           "quant_act", "quant_act_grouped", "quant_act_rms", "quantize_weights", "quantize_weights_grouped",
           "set_decode_engine", "status_string"]
