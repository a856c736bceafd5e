"""Fused, chunked top-K forward-KL distillation loss for B200 (sm_100a).

Modules:
  ckl        -- the Python binding of libckl.so (ChunkedKL, chunked_kl_loss,
                forward_static, VocabGroup / torch_vocab_group / vocab_shards)
  build      -- compiles csrc/ into lib/libckl.so with nvcc for sm_100a
  workloads  -- seeded synthetic inputs of the benchmark workloads

The C ABI is declared in include/ckl.h. Importing this package imports nothing
else, so `python -m chunked_kl_loss_logits_b200.build` does not need torch.
"""
