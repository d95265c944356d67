"""fp64 CPU oracle (test infrastructure only).

Plain numpy restatement of the Summaryformer frame memory and its attention,
written from the model card "GTA world model: weights and inference code".
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg use it; the CUDA library never imports it and it never imports the CUDA
library.
"""
from .kvmemory import (Layout, FrameMemory, attend, attend_bits, attend_memory,
                       softmax_weights, visible_history_mask, masked_history_attend,
                       rotation_cos_sin, rotate_pairs_f64, rotate_keys_bf16, sink_shift,
                       E4M3_MAX, E4M3_NAN, e4m3_decode, e4m3_encode, quantize_e4m3,
                       dequantize_e4m3, TINY, SERVED, SERVED_W16, SCALED)

__all__ = ["Layout", "FrameMemory", "attend", "attend_bits", "attend_memory",
           "softmax_weights", "visible_history_mask", "masked_history_attend",
           "rotation_cos_sin", "rotate_pairs_f64", "rotate_keys_bf16", "sink_shift",
           "E4M3_MAX", "E4M3_NAN", "e4m3_decode", "e4m3_encode", "quantize_e4m3",
           "dequantize_e4m3", "TINY", "SERVED", "SERVED_W16", "SCALED"]
