"""The seeded MoE input recipes, on CPU: shapes and dtypes, determinism, the prefill
layer's +2.0 logit bias on experts 0-3, independent per-expert weight draws, and the
weights' scale."""
import pytest
import torch

from moe_expert_gemm_mxfp4_b200 import inputs


@pytest.mark.parametrize("name,T,E", [("moe_decode", 64, 32), ("moe_prefill", 8192, 32),
                                      ("moe_120b", 4096, 128)])
def test_moe_activation_shapes_and_determinism(name, T, E):
    cfg = inputs.MOE_CONFIGS[name]
    assert (cfg.T, cfg.E, cfg.top_k, cfg.H, cfg.I) == (T, E, 4, 2880, 2880)
    x, logits = inputs.moe_activations(cfg)
    assert x.shape == (T, 2880) and x.dtype == torch.bfloat16
    assert logits.shape == (T, E) and logits.dtype == torch.float32
    x2, logits2 = inputs.moe_activations(cfg)
    assert torch.equal(x.view(torch.int16), x2.view(torch.int16)) and torch.equal(logits, logits2)


def test_prefill_bias_lands_on_experts_0_to_3_only():
    cfg = inputs.MOE_CONFIGS["moe_prefill"]
    _, biased = inputs.moe_activations(cfg)
    _, plain = inputs.moe_activations(inputs.MoEConfig("plain", seed=cfg.seed, T=cfg.T, E=cfg.E))
    assert torch.equal(biased[:, :4], plain[:, :4] + 2.0)
    assert torch.equal(biased[:, 4:], plain[:, 4:])
    # the bias makes the hot experts take far more than their 4/32 share of the pairs
    ids = torch.topk(biased, 4, dim=1).indices
    assert (ids < 4).float().mean() > 0.5


def test_fewer_tokens_are_a_prefix_of_the_layer():
    cfg = inputs.MOE_CONFIGS["moe_decode"]
    x, logits = inputs.moe_activations(cfg)
    xs, ls = inputs.moe_activations(cfg, T=16)
    assert torch.equal(xs.view(torch.int16), x[:16].view(torch.int16))
    # x is drawn first, so the logits of a shorter draw come from other positions of the stream
    assert ls.shape == (16, cfg.E)


def test_expert_weights_are_independent_draws_with_the_recipe_scale():
    cfg = inputs.MoEConfig("small", seed=9, T=8, E=4, H=128, I=64)
    w13, w2 = inputs.expert_weights(cfg, 2)
    assert w13.shape == (128, 128) and w2.shape == (128, 64)
    again, _ = inputs.expert_weights(cfg, 2)
    other, _ = inputs.expert_weights(cfg, 3)
    assert torch.equal(w13, again) and not torch.equal(w13, other)
    assert abs(float(w13.std()) - 0.02) < 0.002 and abs(float(w2.std()) - 0.02) < 0.002
    seeds = {inputs.expert_seed(cfg.seed, e, which) for e in range(cfg.E) for which in (0, 1)}
    assert len(seeds) == 2 * cfg.E
