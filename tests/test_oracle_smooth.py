"""Pins for the oracle's SmoothQuant steps (calibration, factors, fold).

Sources: "探秘Transformer系列之（36）— 大模型量化方案" §1.3 and
"SmoothQuant技术解析：大模型INT8量化的突破与实践" §2.2, §3: the output is
unchanged by Y = (X diag(s)^-1)(diag(s) W); s is chosen per channel offline
so that the smoothed activation channels have similar maxima; the maxima come
from calibration batches.  The factor rule (reading R14 of the oracle) is the
SmoothQuant paper's s_j = amax_j^alpha / wmax_j^(1-alpha).

Pins: hand-worked factors (``tests/golden/smooth_factors.txt``); the balance
property the rule exists for (alpha = 0.5: smoothed activation and weight
channel maxima both equal sqrt(amax * wmax); alpha = 1: every activation
channel max is 1); the output identity through the LayerNorm fold, against
torch float64 LayerNorm and matmul; max over batches equals max over their
concatenation; planted mistakes (on the CPU) break the pins.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.golden.fixtures import load_blocks
from w8a8_post_quantized_b200 import inputs


@pytest.mark.parametrize("block", load_blocks("smooth_factors.txt"))
def test_smooth_factors_hand_examples(block):
    s = oracle.smooth_factors(block["amax"].astype(np.float32), block["wmax"].astype(np.float32),
                              float(block["alpha"][0]))
    np.testing.assert_allclose(s, block["s"].astype(np.float32), rtol=2 ** -23, atol=0)


def _outlier_case(seed=7, T=96, K=64, N=48):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, K)).astype(np.float32)
    x[:, [5, 17, 40]] *= 30.0                       # channel-wise outliers
    gamma = (1 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(K)).astype(np.float32)
    W = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    return x, gamma, beta, W


def _torch_ln(x, gamma, beta, eps):
    return torch.nn.functional.layer_norm(torch.from_numpy(x).double(), (x.shape[1],),
                                          torch.from_numpy(gamma).double(),
                                          torch.from_numpy(beta).double(), eps=eps).numpy()


def test_channel_absmax_matches_numpy_and_accumulates():
    x, *_ = _outlier_case()
    a = oracle.channel_absmax(x)
    np.testing.assert_array_equal(a, np.abs(x).max(0))
    # running max over two batches = max over their concatenation
    b = oracle.channel_absmax(x[50:], oracle.channel_absmax(x[:50]))
    np.testing.assert_array_equal(b, a)


def test_weight_col_absmax_matches_numpy():
    *_, W = _outlier_case()
    np.testing.assert_array_equal(oracle.weight_col_absmax(W), np.abs(W).max(0))


@pytest.mark.parametrize("alpha", [0.5, 1.0, 0.0, 0.8])
def test_smoothing_balances_channel_maxima(alpha):
    """With s_j = amax_j^a / wmax_j^(1-a) the smoothed activation channel max is
    amax_j / s_j = (amax_j wmax_j)^(1-a) and the smoothed weight channel max
    wmax_j s_j = (amax_j wmax_j)^a: for alpha = 0.5 both are sqrt(amax wmax),
    for alpha = 1 every activation max is 1, for alpha = 0 every weight max."""
    x, gamma, beta, W = _outlier_case()
    amax = np.abs(x).max(0).astype(np.float64)
    wmax = np.abs(W).max(0).astype(np.float64)
    s = oracle.smooth_factors(amax.astype(np.float32), wmax.astype(np.float32), alpha).astype(np.float64)
    Ws, _, _ = oracle.smooth_fold(W, s.astype(np.float32))
    act_max = amax / s
    w_max = np.abs(Ws.astype(np.float64)).max(0)
    np.testing.assert_allclose(act_max, amax ** (1 - alpha) * wmax ** (1 - alpha), rtol=1e-6)
    np.testing.assert_allclose(w_max, amax ** alpha * wmax ** alpha, rtol=1e-6)
    # the point of smoothing: the activation channels' spread shrinks
    if alpha > 0:
        assert act_max.max() / act_max.min() < amax.max() / amax.min()


def test_fold_preserves_the_layer_output():
    """LN(x; gamma/s, beta/s) (diag(s) W)^T == LN(x; gamma, beta) W^T up to the
    fp32 rounding of the folded parameters (torch float64 reference)."""
    x, gamma, beta, W = _outlier_case()
    eps = 1e-5
    Wo, go, bo, s, amax = oracle.smooth_ln_linear([x[:40], x[40:]], gamma, beta, eps, W, 0.5)
    ref = _torch_ln(x, gamma, beta, eps) @ W.astype(np.float64).T
    got = _torch_ln(x, go, bo, eps) @ Wo.astype(np.float64).T
    scale = np.abs(_torch_ln(x, gamma, beta, eps)) @ np.abs(W.astype(np.float64)).T
    assert np.max(np.abs(got - ref) / scale) < 1e-6
    # the calibration saw the LayerNorm output, not x
    np.testing.assert_allclose(amax, np.abs(_torch_ln(x, gamma, beta, eps)).max(0), rtol=1e-6)


def test_smoothing_reduces_w8a8_error_on_outlier_channels():
    """The reason for the transform: on activations with outlier channels the
    W8A8 linear's error against the float64 product shrinks."""
    w = inputs.bert_ffn(T=256)
    lin = w.layers[0]
    x = w.x.f32
    eps = w.eps
    ref = _torch_ln(x, w.gamma, w.beta, eps) @ lin.W.astype(np.float64).T
    G = lin.group_rows

    def w8a8(gamma, beta, W):
        xq, st = oracle.ln_quant(x, gamma, beta, eps)
        Wq, sg = oracle.quantize_weights(W, G)
        return oracle.linear(xq, st, Wq, sg, G).astype(np.float64)

    base = np.linalg.norm(w8a8(w.gamma, w.beta, lin.W) - ref) / np.linalg.norm(ref)
    Wo, go, bo, s, _ = oracle.smooth_ln_linear([x], w.gamma, w.beta, eps, lin.W, 0.5)
    smooth = np.linalg.norm(w8a8(go, bo, Wo) - ref) / np.linalg.norm(ref)
    assert smooth < 0.8 * base


SMOOTH_MUTANTS = ["gamma_times_s", "weights_scaled_by_row", "alpha_swapped"]


@pytest.mark.parametrize("mutant", SMOOTH_MUTANTS)
def test_smooth_pins_catch_planted_mistakes(mutant):
    """Plausible mistakes in the smoothing steps, planted on the CPU, break the
    output identity or the balance property."""
    x, gamma, beta, W = _outlier_case()
    eps = 1e-5
    ln = oracle.layernorm(x, gamma, beta, eps)
    amax = oracle.channel_absmax(ln)
    wmax = oracle.weight_col_absmax(W)
    alpha = 0.7
    s = oracle.smooth_factors(amax, wmax, alpha)
    Wo, go, bo = oracle.smooth_fold(W, s, gamma, beta)
    if mutant == "gamma_times_s":                 # activation scaled up instead of down
        go = (gamma.astype(np.float64) * s).astype(np.float32)
        bo = (beta.astype(np.float64) * s).astype(np.float32)
    elif mutant == "weights_scaled_by_row":       # diag(s) applied on the output axis
        N = W.shape[0]
        Wo = (W.astype(np.float64) * np.resize(s, N)[:, None]).astype(np.float32)
    else:                                         # exponents exchanged
        s = oracle.smooth_factors(amax, wmax, 1 - alpha)
        Wo, go, bo = oracle.smooth_fold(W, s, gamma, beta)
    ref = _torch_ln(x, gamma, beta, eps) @ W.astype(np.float64).T
    got = _torch_ln(x, go, bo, eps) @ Wo.astype(np.float64).T
    scale = np.abs(_torch_ln(x, gamma, beta, eps)) @ np.abs(W.astype(np.float64)).T
    identity_ok = np.max(np.abs(got - ref) / scale) < 1e-6
    act_max = amax.astype(np.float64) / s.astype(np.float64)
    balance_ok = np.allclose(act_max, (amax.astype(np.float64) * wmax) ** (1 - alpha), rtol=1e-5)
    assert not (identity_ok and balance_ok)
