"""CPU oracle for the Psi-Spec linear decode step — TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 restatement of what the hot path computes, written from
the method description of "Uno" (hyper.ai page, section "方法": gated LoRA,
linear sampler, rejection-sampling verification of the longest prefix) and the
abstract (chatpaper page: lossless = the base AR distribution is preserved).

Only `tests/`, `__graft_entry__.smoke()` and `bench.py`'s CPU-baseline /
reference legs may import anything from here. It shares no code with the CUDA
path and never consumes a value the CUDA path produced.

Modules
  philox        Philox4x32-10 counter-based generator and the uniform maps.
  gated_linear  y = x W^T + s g (x A^T) Bl^T, and the adapter's gradients
                (dA, dBl) with theta_AR frozen.
  sampling      softmax at temperature T, inverse-CDF draws, the draft
                sampler, acceptance, first rejection, residual and bonus.
  stack         the synthetic decoder stack + LM head used by the step.
  tree          the tree sampler: several drafted blocks verified as a prefix
                tree (multi-candidate rejection sampling along the trie).
  distill       the distillation objective alpha KL + beta TV between teacher
                and student rows, and its gradient w.r.t. the student logits.

Every function states the passage it follows. No function here is "parity
unpinned": each has pins in tests/test_oracle_*.py.
"""
