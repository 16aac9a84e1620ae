"""fp64 CPU oracle (test infrastructure only; see ``oracle.decoder``)."""
from .decoder import (Decoder, argmax_lowest, attend_one, causal_attention, fp16_round,  # noqa: F401
                      kv_head_of, moe_ffn, rmsnorm, rope, silu, softmax,
                      swiglu_ffn, top2_margin, topk_lowest)
