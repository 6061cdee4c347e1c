"""Float64 CPU oracle for structured-mask attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product package imports, links or
runs anything here; only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.
It shares no code, tables or constants with the CUDA path.

Each module writes out the plain definition of one thing the pages describe:

* ``dflash_mask``  -- the DFlash draft-training visibility rule as an
  explicit dense boolean mask (SpecForge issue #452 "flex_attention
  BlockMask incorrectly created with H=num_heads", Problem paragraph;
  SpecForge PR #905 "Fix DFlash attention masking", Motivation list and the
  maintainer's split note on #934).
* ``attention``    -- dense softmax attention with an explicit keep mask and
  additive bias, including the broadcastable 4D mask/bias contract
  (flash-sparse-attention PR #190, Design: "Contract for aux tensors").
* ``attention_grad`` -- the gradients dQ, dK, dV and the broadcast-reduced
  dbias of that attention for an upstream gradient dO (flash-sparse-attention
  PR #190, Changes: mha_bwd and its dbias reductions).
* ``topk``         -- the dynamic top-k keep mask built from an attention bias
  (flash-sparse-attention PR #197, Design and Implementation Notes).
* ``tiles``        -- full / partial / empty classification of 128x128 tiles
  of a dense keep mask (the flex BlockMask notion in SpecForge issue #452).

Every function is pinned by ``tests/test_oracle_*.py`` to hand-worked
fixtures under ``tests/golden/``, to library routines
(``torch.nn.functional.scaled_dot_product_attention``, ``torch.topk``,
``scipy.special.logsumexp``, float64 autograd) on special cases, to central
finite differences of the forward (the gradients), and to brute-force
enumeration on tiny inputs.  No function here is "parity unpinned".
"""
