"""Pins of the oracle's block pieces and of the Conformer block composition.

The composition itself (FFN/2 -> rotary MHSA -> conv module -> FFN/2 ->
LayerNorm) is only partly fixed by the pages; these checks use special weight
settings under which a block reduces to a closed form, so that a dropped term,
a missing 1/2 or a swapped order fails.
"""
import numpy as np
import pytest

import oracle
from conformer_speech_recognition_b200 import synth
from conftest import read_golden, read_golden_rows


def test_layer_norm_invariants():
    rng = np.random.default_rng(0)
    x = rng.normal(3.0, 5.0, size=(6, 32))
    y = oracle.layer_norm(x, np.ones(32), np.zeros(32), 0.0)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-12)
    np.testing.assert_allclose(y.var(axis=1), 1, rtol=1e-12)
    # shift / scale invariance of the normalised part
    np.testing.assert_allclose(oracle.layer_norm(7 * x + 2, np.ones(32), np.zeros(32), 0.0), y, atol=1e-12)
    # affine part
    g, b = rng.normal(size=32), rng.normal(size=32)
    np.testing.assert_allclose(oracle.layer_norm(x, g, b, 0.0), y * g + b, atol=1e-12)


def test_swish_and_glu_closed_forms():
    x = np.linspace(-30, 30, 121)
    s = oracle.swish(x)
    assert oracle.swish(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(s - oracle.swish(-x), x, atol=1e-12)  # x*sig(x) + x*sig(-x) = x
    assert s[-1] == pytest.approx(30.0, rel=1e-12) and abs(s[0]) < 1e-11
    a = np.array([[1.0, -2.0, 0.0, 0.0]])
    np.testing.assert_allclose(oracle.glu(a), [[0.5, -1.0]])
    np.testing.assert_allclose(oracle.glu(np.array([[3.0, 50.0]])), [[3.0]], rtol=1e-12)
    np.testing.assert_allclose(oracle.glu(np.array([[3.0, -50.0]])), [[0.0]], atol=1e-20)


def test_batch_norm_eval_identity_case():
    x = np.random.default_rng(1).normal(size=(4, 3))
    eps = 1e-5
    y = oracle.batch_norm_eval(x, np.ones(3), np.zeros(3), np.zeros(3), np.full(3, 1 - eps), eps)
    np.testing.assert_allclose(y, x, rtol=1e-12)


def _silu_table():
    """x -> (sigma(x), x sigma(x)) from the golden fixture."""
    return {float(x): (float(s), float(y)) for x, s, y in read_golden_rows("activations.txt")}


# Inference BatchNorm, hand-worked cases with var + eps a perfect square:
# gamma (x - mean) / sqrt(var + eps) + beta, per channel.
#   x = 3,  mean = 1,   var + eps = 4,    gamma = 2,  beta = 0.5 ->  2 / 2 * 2 + 0.5 = 2.5
#   x = -1, mean = 0.5, var + eps = 0.25, gamma = 1,  beta = 0   -> -1.5 / 0.5      = -3
#   x = 0,  mean = -2,  var + eps = 16,   gamma = -1, beta = 1   ->  2 / 4 * -1 + 1 = 0.5
_BN_EPS = 1e-5
_BN_CASE = dict(x=[3.0, -1.0, 0.0], mean=[1.0, 0.5, -2.0], var_eps=[4.0, 0.25, 16.0], gamma=[2.0, 1.0, -1.0],
                beta=[0.5, 0.0, 1.0], expected=[2.5, -3.0, 0.5])


def _bn_pin_holds():
    import oracle.gigaam as og
    c = _BN_CASE
    y = og.batch_norm_eval(np.array([c["x"]]), np.array(c["gamma"]), np.array(c["beta"]), np.array(c["mean"]),
                               np.array(c["var_eps"]) - _BN_EPS, _BN_EPS)
    return bool(np.allclose(y[0], c["expected"], rtol=0, atol=1e-12))


def test_batch_norm_eval_hand_cases():
    assert _bn_pin_holds()


def test_batch_norm_folded_equals_unfolded():
    """BatchNorm after the depthwise conv folds into the conv's weight and bias:
    w' = w g / sqrt(v + eps), b' = (b - mu) g / sqrt(v + eps) + beta."""
    rng = np.random.default_rng(11)
    T, d, K = 9, 5, 5
    x = rng.normal(size=(T, d))
    w, b = rng.normal(size=(d, 1, K)), rng.normal(size=d)
    g, beta = rng.normal(1.0, 0.3, size=d), rng.normal(size=d)
    mu, var = rng.normal(size=d), rng.uniform(0.2, 3.0, size=d)
    unfolded = oracle.batch_norm_eval(oracle.depthwise_conv1d(x, w, b), g, beta, mu, var, _BN_EPS)
    sc = g / np.sqrt(var + _BN_EPS)
    folded = oracle.depthwise_conv1d(x, w * sc[:, None, None], (b - mu) * sc + beta)
    np.testing.assert_allclose(unfolded, folded, rtol=0, atol=1e-12)


def _ffn_pin_holds():
    """linear1 = [I; 0], linear2 = [I | 0], zero biases: FFN(u) = SiLU(u), compared
    with the fixture's SiLU values."""
    tab = _silu_table()
    d, f = 4, 8
    u = np.array([[1.0, -1.0, 2.0, 0.5], [-2.0, 3.0, -0.5, 1.0]])
    W = {"f.linear1.weight": np.vstack([np.eye(d), np.zeros((f - d, d))]), "f.linear1.bias": np.zeros(f),
         "f.linear2.weight": np.hstack([np.eye(d), np.zeros((d, f - d))]), "f.linear2.bias": np.zeros(d)}
    y = oracle.feed_forward(u, W, "f", np.float64)
    expected = np.vectorize(lambda v: tab[float(v)][1])(u)
    return bool(np.allclose(y, expected, rtol=0, atol=1e-15))


def test_feed_forward_activation_is_silu():
    assert _ffn_pin_holds()


def _conv_module_pin_holds():
    """Conv module with a non-identity BatchNorm.  pointwise1 = [I; 0] (GLU gate 0,
    so sigma = 1/2), depthwise = centre tap 1 and bias 0, pointwise2 = I, and per
    channel a BatchNorm chosen so that BN(u / 2) is 1, -1 and 2:
      ch0: u = 4  -> 2   -> (2 - 1) / 2 * 2         = 1  -> SiLU(1)
      ch1: u = -2 -> -1  -> (-1 - 0) / 1 * 1        = -1 -> SiLU(-1)
      ch2: u = 1  -> 0.5 -> (0.5 - 0.5) / 0.5 + 2   = 2  -> SiLU(2)
    BatchNorm after SiLU, or no BatchNorm, or another activation gives other values."""
    tab = _silu_table()
    d, K, T = 3, 5, 3
    cfg, W = _zero_layer_weights(d, 8, K)
    p = "layers.0.conv"
    W[p + ".pointwise1.weight"] = np.concatenate([np.eye(d), np.zeros((d, d))])[:, :, None]
    W[p + ".depthwise.weight"][:, 0, K // 2] = 1.0
    W[p + ".pointwise2.weight"] = np.eye(d)[:, :, None]
    W[p + ".bn.running_mean"] = np.array([1.0, 0.0, 0.5])
    W[p + ".bn.running_var"] = np.array([4.0, 1.0, 0.25]) - cfg["bn_eps"]
    W[p + ".bn.weight"] = np.array([2.0, 1.0, 1.0])
    W[p + ".bn.bias"] = np.array([0.0, 0.0, 2.0])
    u = np.tile(np.array([[4.0, -2.0, 1.0]]), (T, 1))
    y = oracle.conv_module(u, W, p, cfg, np.float64)
    expected = np.tile(np.array([[tab[1.0][1], tab[-1.0][1], tab[2.0][1]]]), (T, 1))
    return bool(np.allclose(y, expected, rtol=0, atol=1e-14))


def test_conv_module_batchnorm_before_silu():
    assert _conv_module_pin_holds()


def _relu(x):
    return np.maximum(x, 0.0)


def _identity(x):
    return x


def _gelu_tanh(x):
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))


@pytest.mark.parametrize("mutant", [_relu, _identity, _gelu_tanh], ids=["relu", "identity", "gelu"])
def test_activation_pins_catch_a_wrong_activation(monkeypatch, mutant):
    """A mistake planted in the oracle (another activation in place of SiLU) is
    caught by the FFN and conv-module pins."""
    import oracle.gigaam as og
    monkeypatch.setattr(og, "swish", mutant)
    assert not _ffn_pin_holds()
    assert not _conv_module_pin_holds()


def _bn_x_plus_mean(x, gamma, beta, mean, var, eps):
    return (x + mean) / np.sqrt(var + eps) * gamma + beta


def _bn_times_root(x, gamma, beta, mean, var, eps):
    return (x - mean) * np.sqrt(var + eps) * gamma + beta


def _bn_eps_outside(x, gamma, beta, mean, var, eps):
    return (x - mean) / (np.sqrt(var) + eps) * gamma + beta


def _bn_missing(x, gamma, beta, mean, var, eps):
    return x


@pytest.mark.parametrize("mutant", [_bn_x_plus_mean, _bn_times_root, _bn_eps_outside, _bn_missing],
                         ids=["x_plus_mean", "times_root", "eps_outside_root", "missing"])
def test_batchnorm_pins_catch_a_wrong_formula(monkeypatch, mutant):
    import oracle.gigaam as og
    monkeypatch.setattr(og, "batch_norm_eval", mutant)
    assert not _bn_pin_holds()
    assert not _conv_module_pin_holds()


def test_depthwise_conv_vs_numpy_correlate():
    rng = np.random.default_rng(2)
    T, d, K = 11, 3, 5
    x = rng.normal(size=(T, d))
    w = rng.normal(size=(d, 1, K))
    b = rng.normal(size=d)
    y = oracle.depthwise_conv1d(x, w, b)
    for c in range(d):
        ref = np.correlate(np.pad(x[:, c], (2, 2)), w[c, 0], mode="valid") + b[c]
        np.testing.assert_allclose(y[:, c], ref, rtol=1e-12)


def _zero_layer_weights(d, f, K, H=2):
    cfg = dict(n_layers=1, d_model=d, n_heads=H, ffn_dim=f, conv_kernel=K, n_mels=64, n_fft=320,
               win=320, hop=160, sub_kernel=5, n_classes=5, rope_base=5000.0, ln_eps=1e-5,
               bn_eps=1e-5, precision="fp32")
    W = {}
    for name, shape in synth.weight_shapes(cfg).items():
        W[name] = np.zeros(shape)
    for name in W:
        if name.endswith("norm.weight") or name.endswith("norm_out.weight") or name.endswith("bn.weight") \
                or name.endswith("running_var"):
            W[name] = np.ones_like(W[name])
    W["layers.0.conv.bn.running_var"][:] = 1.0 - cfg["bn_eps"]
    return cfg, W


def test_layer_with_zero_weights_is_final_layernorm():
    d, T = 8, 5
    cfg, W = _zero_layer_weights(d, 16, 3)
    x = np.random.default_rng(3).normal(size=(T, d))
    y = oracle.conformer_layer(x, W, 0, cfg)
    np.testing.assert_allclose(y, oracle.layer_norm(x, np.ones(d), np.zeros(d), 1e-5), atol=1e-12)


@pytest.mark.parametrize("name,weight", [("layers.0.ffn1.linear2.bias", 0.5),
                                         ("layers.0.ffn2.linear2.bias", 0.5),
                                         ("layers.0.attn.linear_out.bias", 1.0),
                                         ("layers.0.conv.pointwise2.bias", 1.0)])
def test_residual_weights(name, weight):
    """Only one output bias c set: the block returns LN(x + weight * c)."""
    d, T = 8, 4
    cfg, W = _zero_layer_weights(d, 16, 3)
    c = np.random.default_rng(4).normal(size=d)
    W[name] = c
    x = np.random.default_rng(5).normal(size=(T, d))
    y = oracle.conformer_layer(x, W, 0, cfg)
    np.testing.assert_allclose(y, oracle.layer_norm(x + weight * c, np.ones(d), np.zeros(d), 1e-5), atol=1e-12)


def test_conv_module_closed_form():
    """pointwise1 = [I; 0] (gate 0 -> sigmoid 1/2), depthwise = one tap that
    reads the next frame, BN identity, pointwise2 = I:
    conv(u)[t] = swish(u[t+1] / 2) with a zero frame after the clip."""
    d, T, K = 4, 6, 5
    cfg, W = _zero_layer_weights(d, 8, K)
    p = "layers.0.conv"
    W[p + ".pointwise1.weight"] = np.concatenate([np.eye(d), np.zeros((d, d))])[:, :, None]
    W[p + ".depthwise.weight"][:, 0, K // 2 + 1] = 1.0
    W[p + ".pointwise2.weight"] = np.eye(d)[:, :, None]
    u = np.random.default_rng(6).normal(size=(T, d))
    y = oracle.conv_module(u, W, p, cfg, np.float64)
    shifted = np.concatenate([u[1:], np.zeros((1, d))]) * 0.5
    np.testing.assert_allclose(y, oracle.swish(shifted), atol=1e-12)


def test_block_order_ffn_before_attention():
    """FFN1's output bias enters the attention's V path: with V = I and uniform
    attention the MHSA output is the clip mean of LN(x + c/2), which differs
    from the mean of LN(x) when the order is wrong."""
    d, T = 8, 5
    cfg, W = _zero_layer_weights(d, 16, 3)
    rng = np.random.default_rng(7)
    c = rng.normal(size=d)
    W["layers.0.ffn1.linear2.bias"] = c
    W["layers.0.attn.linear_v.weight"] = np.eye(d)
    W["layers.0.attn.linear_out.weight"] = np.eye(d)
    x = rng.normal(size=(T, d))
    y = oracle.conformer_layer(x, W, 0, cfg)
    x1 = x + 0.5 * c
    u = oracle.layer_norm(x1, np.ones(d), np.zeros(d), 1e-5)
    x2 = x1 + u.mean(axis=0)
    np.testing.assert_allclose(y, oracle.layer_norm(x2, np.ones(d), np.zeros(d), 1e-5), atol=1e-12)


def _param_count(cfg):
    inv = oracle.oracle_weight_inventory(cfg)
    return {k: int(np.prod(s)) for k, s in inv.items() if "running_" not in k}


def test_parameter_totals_match_pages():
    g = read_golden("params.txt")
    large = synth.model_config(dict(synth.LARGE, conv_kernel=5), 80, "fp16")
    n = _param_count(large)
    total = sum(n.values())
    ffn = sum(v for k, v in n.items() if ".ffn" in k and "norm" not in k)
    attn = sum(v for k, v in n.items() if ".attn.linear" in k)
    conv = sum(v for k, v in n.items() if ".conv." in k and "norm" not in k)
    assert round(ffn / 1e6, 2) == float(g["large_ffn_millions"])
    assert abs(total / 1e6 - float(g["large_total_millions"])) < 0.1
    assert round(100 * attn / total, 1) == float(g["large_attention_share_pct"])
    assert round(100 * conv / total, 1) == float(g["large_conv_share_pct"])
    v3 = synth.model_config(synth.V3, 34, "fp16")
    mib = 2 * sum(_param_count(v3).values()) / 2 ** 20
    assert float(g["v3_fp16_mb_min"]) <= mib <= float(g["v3_fp16_mb_max"])


def test_generator_matches_oracle_inventory():
    for model in (synth.V3, synth.LARGE):
        cfg = synth.model_config(dict(model, n_layers=2), 257, "fp16")
        gen = {k: v for k, v in synth.weight_shapes(cfg).items() if not k.startswith("frontend.")}
        assert gen == oracle.oracle_weight_inventory(cfg)
