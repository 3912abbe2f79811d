"""CPU oracle (test infrastructure only; see dma_oracle's header)."""
from .dma_oracle import (MIN_DTYPE, softplus, dt_scores64, dt_scores, dynamic_mask_rows,
                         kept_mask, composite_key, threshold_row, thresholds, attention_rows,
                         prefill_rows, prefill, decode_step, rms_norm, rope_angles, rope, prologue, cdmoe_logits, cdmoe_route,
                         cdmoe_experts, cdmoe, prefill_backward)
