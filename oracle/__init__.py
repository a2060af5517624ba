"""Float64 CPU oracle of the pretraining forward+backward step.

Test infrastructure: only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline may import it.  The product path never touches it.
"""
from .model import (RMS_EPS, layout, views, rmsnorm, rmsnorm_backward, rope_tables, rope,
                    rope_backward, attention, attention_backward, softcap, lm_head_loss,
                    step, position_losses, forward_logits)
from .optim import adamw_step
from .decode import prefill, decode_step

__all__ = ["RMS_EPS", "layout", "views", "rmsnorm", "rmsnorm_backward", "rope_tables", "rope",
           "rope_backward", "attention", "attention_backward", "softcap", "lm_head_loss",
           "step", "position_losses", "forward_logits", "adamw_step",
           "prefill", "decode_step"]
