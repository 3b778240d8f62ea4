"""CPU oracle for the DFlash draft cycle — TEST INFRASTRUCTURE ONLY.

A plain, slow, float64 NumPy restatement of what one draft cycle computes,
written from the DFlash pages and kept free of any blocking, fusion or
reordering beyond what the definitions state. It shares no code with the CUDA
path and never imports it. Only the test-suite, the smoke check and the
benchmark's CPU-baseline leg may use it; the product path must not.

Modules
  dflash  -- feature fusion + KV injection, the block drafter, greedy verify
  target  -- a tiny causal target model, greedy autoregressive decoding and the
             speculative loop (for the lossless check)
  sampling -- sampled (temperature > 0) verification and Gumbel-max drafting
  philox  -- the Philox4x32-10 counter-based generator of the draft noise
  policy  -- acceptance counts and the dynamic block-size choice

Parity status per function (what pins each one, see tests/test_oracle_*.py):
  rms_norm, silu, apply_rope, block_attention, drafter_layer, inject,
  draft_block                 pinned (closed forms, invariants, library routines)
  greedy_argmax, verify       pinned (brute force, hand-worked golden cases)
  TinyTarget, greedy_decode,
  spec_generate               pinned (library decoder, lossless invariant)
  softmax_t, sample_index,
  sampled_verify,
  gumbel_sample, gumbel_draft pinned (exact first-token marginal, special cases,
                              greedy limit, Markov-chain loop, softmax frequencies)
  philox4x32_10, draft_uniforms
                              pinned (published known-answer vectors, layout, moments)
  acceptance_counts, BlockPolicy
                              pinned (hand-worked counts, geometric closed form,
                              brute-force enumeration, simulated convergence, limits)
"""
