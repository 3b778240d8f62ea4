"""The tiny drafter / tiny target pair used by the lossless checks: fp32, the
drafter shares the target's embedding, which is also the (tied) LM head."""
from block_diffusion_speculative_cycle_b200 import synth

TARGET_CFG = synth.TINY.replace(n_layers=4)


def tiny_pair(seed=0):
    tw = synth.make_drafter_weights(TARGET_CFG, seed=1000 + seed, share_embed_lm_head=True)
    dw = synth.make_drafter_weights(synth.TINY, seed=seed, embed=tw["embed"], share_embed_lm_head=True)
    return tw, dw
