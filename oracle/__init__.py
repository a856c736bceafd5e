"""fp64 CPU oracle for the fused top-K forward-KL loss (test infrastructure only).

Imported by the tests, by the smoke check and by the benchmark's CPU-baseline leg.
The library under chunked_kl_loss_logits_b200/ never imports it.
"""
from .ckl_oracle import (dW_rows, fwd_bwd, grad_logits, logsumexp, merged_probs, sampled_rows,  # noqa: F401
                         topk_cache,
                         student_logits, teacher_probs, token_loss, token_scale)
