"""Pins for the oracle's LLM.int8() mixed-precision decomposition
("探秘Transformer系列之（36）— 大模型量化方案" §1.1, reading R16 of the oracle).

Pins: hand-worked outlier detection (``tests/golden/outlier_columns.txt``);
the fp16 rounding of the outlier operands against numpy's IEEE float16
conversion; the two special cases that reduce to known results (no outlier:
exactly the plain W8A8 linear; every column an outlier: exactly the fp16
product plus bias, the INT8 part being all zero codes); the purpose of the
method (on activations with large outlier columns the decomposed result is
far closer to the float64 product than the plain W8A8 one); planted mistakes
(on the CPU) break these pins.
"""
import numpy as np
import pytest

import oracle
from tests.golden.fixtures import load_blocks


@pytest.mark.parametrize("block", load_blocks("outlier_columns.txt"))
def test_outlier_columns_hand_examples(block):
    idx, n = oracle.outlier_columns(block["amax"].astype(np.float32), float(block["threshold"][0]),
                                    int(block["max_o"][0]))
    np.testing.assert_array_equal(idx, block["idx"].astype(np.int32))
    assert n == int(block["count"][0])


def test_outlier_operands_round_to_fp16_like_numpy():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(2000) * 10 ** rng.uniform(-9, 5, 2000),
                        [0.0, -0.0, 65504.0, 65519.9, 65520.0, -70000.0, 2 ** -24, 2 ** -25, 3 * 2 ** -26,
                         1 + 2 ** -11, 1 + 3 * 2 ** -11, 2049.0, 2051.0]]).astype(np.float32)
    a = v.reshape(-1, 1)
    W = np.ones((1, 1), np.float32)
    got = oracle.outlier_product(a, W, np.array([0], np.int32))[:, 0]
    with np.errstate(over="ignore"):                  # 65520 and beyond become inf, as intended
        want = v.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(got, want)


def _case(seed=11, T=64, K=128, N=96, G=16, scale=40.0, n_out=3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, K)).astype(np.float32)
    cols = rng.permutation(K)[:n_out]
    x[:, cols] *= scale
    gamma = (1 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(K)).astype(np.float32)
    W = (0.05 * rng.standard_normal((N, K))).astype(np.float32)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    Wq, sg = oracle.quantize_weights(W, G)
    return x, gamma, beta, W, Wq, sg, G, bias, np.sort(cols)


def test_no_outlier_is_the_plain_w8a8_linear():
    x, gamma, beta, W, Wq, sg, G, bias, _ = _case(scale=1.0)
    y, idx, n = oracle.int8_decomposed_ln_linear(x, gamma, beta, 1e-5, W, Wq, sg, G, bias, threshold=np.inf)
    assert n == 0 and idx.size == 0
    xq, st = oracle.ln_quant(x, gamma, beta, 1e-5)
    np.testing.assert_array_equal(y, oracle.linear(xq, st, Wq, sg, G, bias))


def test_all_columns_outliers_is_the_fp16_product():
    x, gamma, beta, W, Wq, sg, G, bias, _ = _case()
    K = x.shape[1]
    y, idx, n = oracle.int8_decomposed_ln_linear(x, gamma, beta, 1e-5, W, Wq, sg, G, bias, threshold=0.0,
                                                 max_o=K)
    assert n == K
    a = oracle.layernorm(x, gamma, beta, 1e-5)
    ref = (a.astype(np.float16).astype(np.float64) @ W.astype(np.float16).astype(np.float64).T
           + bias.astype(np.float64))
    np.testing.assert_allclose(y, ref.astype(np.float32), rtol=0, atol=0)


def test_decomposition_detects_the_planted_columns_and_beats_plain_w8a8():
    x, gamma, beta, W, Wq, sg, G, bias, cols = _case()
    y, idx, n = oracle.int8_decomposed_ln_linear(x, gamma, beta, 1e-5, W, Wq, sg, G, bias)
    a = oracle.layernorm(x, gamma, beta, 1e-5)
    # the planted columns dominate the LayerNorm output and are exactly the ones found
    np.testing.assert_array_equal(idx, cols)
    ref = a.astype(np.float64) @ W.astype(np.float64).T + bias
    xq, st = oracle.ln_quant(x, gamma, beta, 1e-5)
    plain = oracle.linear(xq, st, Wq, sg, G, bias)
    err_d = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    err_p = np.linalg.norm(plain - ref) / np.linalg.norm(ref)
    assert err_d < 0.5 * err_p


MUTANTS = ["outliers_left_in_int8_part", "outlier_columns_shifted", "outlier_part_dropped"]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_decomposition_pins_catch_planted_mistakes(mutant):
    """Each plausible mistake, planted on the CPU, breaks the all-outliers
    closed form or the accuracy property."""
    x, gamma, beta, W, Wq, sg, G, bias, cols = _case()
    K = x.shape[1]
    a = oracle.layernorm(x, gamma, beta, 1e-5)

    def run(threshold, max_o):
        idx, n = oracle.outlier_columns(oracle.channel_absmax(a), threshold, max_o)
        a_in = a.copy()
        if mutant != "outliers_left_in_int8_part":
            a_in[:, idx] = 0.0
        xq, st = oracle.quantize_rows(a_in)
        used = (idx + 1) % K if mutant == "outlier_columns_shifted" else idx
        add = None if mutant == "outlier_part_dropped" else oracle.outlier_product(a, W, used)
        return oracle.dequant_add(oracle.gemm_i32(xq, Wq), st, sg, G, add, bias)

    y_all = run(0.0, K)
    ref_all = (a.astype(np.float16).astype(np.float64) @ W.astype(np.float16).astype(np.float64).T
               + bias.astype(np.float64)).astype(np.float32)
    closed_ok = np.array_equal(y_all, ref_all)
    ref = a.astype(np.float64) @ W.astype(np.float64).T + bias
    y = run(oracle.LLM_INT8_ALPHA, 8)
    xq, st = oracle.ln_quant(x, gamma, beta, 1e-5)
    plain = oracle.linear(xq, st, Wq, sg, G, bias)
    better = np.linalg.norm(y - ref) < 0.5 * np.linalg.norm(plain - ref)
    assert not (closed_ok and better)
