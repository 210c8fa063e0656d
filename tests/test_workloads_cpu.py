"""The seeded input generator follows its stated recipe (CPU only).

The five layers (shapes, storage types, activation laws, outlier fractions, weight
spreads) are checked on the table itself, and the recipe on small layers drawn with
each law: determinism, independence of the substreams, the outlier channels and their
multiplier, the sign of the non-negative law, and the weight spread.
"""
import numpy as np
import pytest
import torch

from workloads import (WORKLOADS, LayerSpec, as_f32_numpy, custom_spec, generate, generate_down, generate_qkv,
                       outlier_channels)


def test_the_five_layers():
    shapes = {name: (s.M, s.K, s.N, s.dtype, s.group, s.n_grid) for name, s in WORKLOADS.items()}
    assert shapes == {
        "single_linear_128x256x256_f32": (128, 256, 256, "f32", 128, 20),
        "llama7b_attn_proj_4096x4096x4096": (4096, 4096, 4096, "bf16", 128, 20),
        "llama7b_mlp_gate_up_4096x4096x22016": (4096, 4096, 22016, "bf16", 128, 20),
        "llama7b_mlp_down_4096x11008x4096": (4096, 11008, 4096, "bf16", 128, 20),
        "llama70b_mlp_gate_up_16384x8192x57344": (16384, 8192, 57344, "bf16", 128, 20),
    }
    down = WORKLOADS["llama7b_mlp_down_4096x11008x4096"]
    assert (down.law, down.sigma, down.outlier_mult, down.w_std) == ("abs_normal", 1.0, 50.0, 0.015)
    for name in ("single_linear_128x256x256_f32", "llama7b_attn_proj_4096x4096x4096",
                 "llama7b_mlp_gate_up_4096x4096x22016"):
        s = WORKLOADS[name]
        assert (s.law, s.sigma, s.outlier_mult, s.w_std, s.seed) == ("normal", 0.5, 20.0, 0.02, 0)
    big = WORKLOADS["llama70b_mlp_gate_up_16384x8192x57344"]
    assert (big.law, big.sigma, big.outlier_mult, big.w_std) == ("normal", 0.5, 20.0, 0.01)
    # 1 % outlier channels: 3, 41, 41, 110 and 82 of them
    assert [len(outlier_channels(s)) for s in WORKLOADS.values()] == [3, 41, 41, 110, 82]


def test_generation_is_a_pure_function_of_the_spec():
    spec = custom_spec(64, 256, 128, seed=7)
    X1, W1 = generate(spec)
    X2, W2 = generate(spec)
    assert torch.equal(X1.view(torch.int16), X2.view(torch.int16))
    assert torch.equal(W1.view(torch.int16), W2.view(torch.int16))
    X3, W3 = generate(custom_spec(64, 256, 128, seed=8))
    assert not torch.equal(X1, X3) and not torch.equal(W1, W3)
    # one substream per tensor: the weights do not depend on the number of tokens
    _, W4 = generate(custom_spec(32, 256, 128, seed=7))
    assert torch.equal(W1.view(torch.int16), W4.view(torch.int16))


@pytest.mark.parametrize("law,mult", [("normal", 20.0), ("abs_normal", 50.0)])
def test_outlier_channels_carry_the_multiplier(law, mult):
    K = 1200
    spec = LayerSpec(f"t_{law}", 4096, K, 8, "f32", law, 0.5, mult, 0.02, 128, 20, 3)
    X, _ = generate(spec)
    x = as_f32_numpy(X).astype(np.float64)
    rms = np.sqrt((x * x).mean(axis=0))
    out = outlier_channels(spec)
    assert len(out) == 12
    rest = np.setdiff1d(np.arange(K), out)
    # the outliers' typical magnitude is the multiplier times the others' (log-normal(0, 0.5)
    # magnitudes: the medians of the two sets differ by about `mult`)
    ratio = np.median(rms[out]) / np.median(rms[rest])
    assert 0.4 * mult < ratio < 2.5 * mult
    # and every outlier column stands above the bulk of the others
    assert np.min(rms[out]) > np.median(rms[rest])
    if law == "abs_normal":
        assert (x >= 0).all()
    else:
        assert (x < 0).mean() > 0.45


def test_weight_spread_and_storage_types():
    spec = custom_spec(16, 512, 1024, seed=11, w_std=0.015)
    X, W = generate(spec)
    assert X.dtype == torch.bfloat16 and W.dtype == torch.bfloat16
    w = as_f32_numpy(W).astype(np.float64)
    assert abs(w.std() - 0.015) < 0.0005 and abs(w.mean()) < 0.0005
    Xf, Wf = generate(custom_spec(16, 512, 1024, dtype="f32", seed=11, w_std=0.015))
    assert Xf.dtype == torch.float32 and Wf.dtype == torch.float32
    # the bf16 layer is the fp32 one rounded to nearest even
    assert torch.equal(W.view(torch.int16), Wf.to(torch.bfloat16).view(torch.int16))


def test_down_projection_is_drawn_from_its_own_substream():
    spec = custom_spec(16, 256, 128, seed=4)
    X, W = generate(spec)
    D = generate_down(spec, 96)
    assert D.shape == (64, 96) and D.dtype == torch.bfloat16
    X2, W2 = generate(spec)
    assert torch.equal(W.view(torch.int16), W2.view(torch.int16))
    with pytest.raises(ValueError):  # [gate | up] needs an even column count
        generate_down(LayerSpec("odd", 16, 256, 135, "bf16", "normal", 0.5, 20.0, 0.02), 96)


def test_qkv_projections_extend_the_query_layer():
    """An attention block's [W_q | W_k | W_v]: W_q is the layer's own W, W_k and W_v come from
    their own substreams with the layer's weight spread, and X is unchanged."""
    spec = custom_spec(32, 256, 256, seed=11)
    X, W = generate(spec)
    Wqkv = generate_qkv(spec)
    assert Wqkv.shape == (256, 768) and Wqkv.dtype == torch.bfloat16
    assert torch.equal(Wqkv[:, :256], W)
    Wk, Wv = as_f32_numpy(Wqkv[:, 256:512]), as_f32_numpy(Wqkv[:, 512:])
    for part in (Wk, Wv):
        assert abs(float(part.std()) - spec.w_std) < 0.05 * spec.w_std
    assert not np.array_equal(Wk, Wv) and not np.array_equal(Wk, as_f32_numpy(W))
    assert torch.equal(generate(spec)[0], X)
    with pytest.raises(ValueError):
        generate_qkv(custom_spec(16, 256, 512, seed=1))
