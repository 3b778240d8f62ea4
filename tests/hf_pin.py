"""Builds the `transformers` Llama modules from a weight dict, so that the
oracle can be pinned against an independent library implementation of the
same pieces (pre-norm RMSNorm, rotate-half RoPE, grouped-query attention,
SwiGLU MLP). The library computes RMSNorm statistics, RoPE tables and softmax
in fp32 even for fp64 inputs, so comparisons against it use ~1e-5 tolerances."""
import torch


def llama_config(cfg, n_layers):
    from transformers import LlamaConfig
    c = LlamaConfig(hidden_size=cfg.hidden, intermediate_size=cfg.intermediate, num_hidden_layers=n_layers,
                    num_attention_heads=cfg.n_q_heads, num_key_value_heads=cfg.n_kv_heads,
                    head_dim=cfg.head_dim, vocab_size=cfg.vocab, rope_theta=cfg.rope_theta,
                    rms_norm_eps=cfg.rms_eps, attention_bias=False, mlp_bias=False,
                    tie_word_embeddings=False, max_position_embeddings=1 << 16)
    c._attn_implementation = "eager"
    return c


def _t(a):
    return torch.as_tensor(a).to(torch.float64)


def load_layer(layer, lw):
    with torch.no_grad():
        layer.input_layernorm.weight.copy_(_t(lw["attn_norm"]))
        layer.post_attention_layernorm.weight.copy_(_t(lw["mlp_norm"]))
        layer.self_attn.q_proj.weight.copy_(_t(lw["wq"]))
        layer.self_attn.k_proj.weight.copy_(_t(lw["wk"]))
        layer.self_attn.v_proj.weight.copy_(_t(lw["wv"]))
        layer.self_attn.o_proj.weight.copy_(_t(lw["wo"]))
        layer.mlp.gate_proj.weight.copy_(_t(lw["wgate"]))
        layer.mlp.up_proj.weight.copy_(_t(lw["wup"]))
        layer.mlp.down_proj.weight.copy_(_t(lw["wdown"]))


def decoder_layers(cfg, weights):
    from transformers.models.llama import modeling_llama as ml
    c = llama_config(cfg, len(weights["layers"]))
    layers = []
    for l, lw in enumerate(weights["layers"]):
        layer = ml.LlamaDecoderLayer(c, layer_idx=l).double().eval()
        load_layer(layer, lw)
        layers.append(layer)
    rot = ml.LlamaRotaryEmbedding(c).double()
    return c, layers, rot


def causal_lm(cfg, weights):
    from transformers.models.llama import modeling_llama as ml
    c = llama_config(cfg, len(weights["layers"]))
    m = ml.LlamaForCausalLM(c).double().eval()
    with torch.no_grad():
        m.model.embed_tokens.weight.copy_(_t(weights["embed"]))
        m.lm_head.weight.copy_(_t(weights["lm_head"]))
        m.model.norm.weight.copy_(_t(weights["final_norm"]))
    for l, lw in enumerate(weights["layers"]):
        load_layer(m.model.layers[l], lw)
    return m
