"""CPU oracle (float64) for the ARCHead packed LM-head.

TEST INFRASTRUCTURE: imported only by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py.  It is independent of the CUDA library.
"""
from .archead_oracle import *  # noqa: F401,F403
from .archead_oracle import (bf16_decode, build_packed_head, component_bytes, correction_factors,  # noqa: F401
                             damped_metric, dequantize, dequantized_factors, fp16_decode, fp16_encode,
                             logits, logits_factored, lse_argmax_ce, metric_objective, packed_bytes,
                             quantize_symmetric, tolerance, truncated_svd, w_hat_rows, QRANGE)
