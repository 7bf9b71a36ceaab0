"""Pins for the oracle's K-axis weight groups (the group-wise paragraph of
"[2022 NeurIPS] ZeroQuant: Efficient and Affordable Post-Training
Quantization for Large-Scale Transformers" and "探秘Transformer系列之（36）—
大模型量化方案" §1.2.2 read along the input axis, reading R17 of the oracle).

Pins: hand-worked quantization and linear outputs
(``tests/golden/kgroup_linear.txt``); one group per row reduces exactly to
the per-channel weight quantizer; the grouped linear equals "dequantize, then
matmul" computed by numpy in float64 (the fake-quantization form of
"Integer Quantization: Deep Dive", 量化模拟), with GeLU from scipy's erf;
quantizer invariants; the purpose of the method (weights whose input
channels differ in range lose far less to K-axis groups than to per-row
scales); planted mistakes (on the CPU) break the hand-worked example.
"""
import numpy as np
import pytest
from scipy.special import erf

import oracle
from tests.golden.fixtures import load_blocks

BLOCKS = load_blocks("kgroup_linear.txt")


def _case(b):
    W = np.atleast_2d(b["W"]).astype(np.float32)
    G = int(b["G"][0])
    xq = np.atleast_2d(b["xq"]).astype(np.int8)
    return W, G, xq, b["s_tok"].astype(np.float32), b["bias"].astype(np.float32)


@pytest.mark.parametrize("block", BLOCKS)
def test_kgroup_hand_examples(block):
    W, G, xq, st, bias = _case(block)
    N, K = W.shape
    Wq, sw = oracle.quantize_weights_kgroups(W, G)
    np.testing.assert_array_equal(Wq, np.atleast_2d(block["Wq"]).astype(np.int8))
    np.testing.assert_array_equal(sw, block["s_w"].astype(np.float32).reshape(N, K // G))
    y = oracle.linear_kgroups(xq, st, Wq, sw, G, bias)
    np.testing.assert_array_equal(y, np.atleast_2d(block["y"]).astype(np.float32).reshape(y.shape))


@pytest.mark.parametrize("N,K", [(16, 64), (7, 96), (33, 256)])
def test_one_group_per_row_is_the_per_channel_quantizer(N, K):
    rng = np.random.default_rng(N * K)
    W = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    Wq, sw = oracle.quantize_weights_kgroups(W, K)
    Wq1, s1 = oracle.quantize_weights(W, 1)
    np.testing.assert_array_equal(Wq, Wq1)
    np.testing.assert_array_equal(sw[:, 0], s1)
    xq = rng.integers(-127, 128, (9, K)).astype(np.int8)
    st = rng.uniform(0.001, 0.1, 9).astype(np.float32)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    for act in (oracle.ACT_NONE, oracle.ACT_GELU):
        y = oracle.linear_kgroups(xq, st, Wq, sw, K, bias, act)
        y1 = oracle.linear(xq, st, Wq1, s1, 1, bias, act)
        # both round a double result once; the doubles differ only in rounding order
        np.testing.assert_array_max_ulp(y, y1, maxulp=1)


def _fake_quant(xq, st, Wq, sw, G, bias, act):
    """Dequantize both operands, then one float64 matmul (numpy)."""
    xd = st.astype(np.float64)[:, None] * xq.astype(np.float64)
    wd = np.repeat(sw.astype(np.float64), G, axis=1) * Wq.astype(np.float64)
    v = xd @ wd.T + bias.astype(np.float64)
    mag = np.abs(xd) @ np.abs(wd).T + np.abs(bias.astype(np.float64))
    if act == oracle.ACT_GELU:
        v = 0.5 * v * (1.0 + erf(v / np.sqrt(2.0)))
    return v, mag


@pytest.mark.parametrize("T,K,N,G,act", [(5, 64, 24, 16, 0), (12, 256, 40, 32, 1), (3, 384, 17, 128, 0),
                                         (8, 96, 8, 1, 1)])
def test_linear_is_dequantize_then_matmul(T, K, N, G, act):
    rng = np.random.default_rng(T + K + N + G)
    W = (0.02 * rng.standard_normal((N, K)) * np.exp(rng.uniform(-2, 2, (1, K)))).astype(np.float32)
    Wq, sw = oracle.quantize_weights_kgroups(W, G)
    assert sw.shape == (N, K // G)
    xq = rng.integers(-127, 128, (T, K)).astype(np.int8)
    st = rng.uniform(0.001, 0.1, T).astype(np.float32)
    bias = (0.1 * rng.standard_normal(N)).astype(np.float32)
    y = oracle.linear_kgroups(xq, st, Wq, sw, G, bias, act).astype(np.float64)
    ref, mag = _fake_quant(xq, st, Wq, sw, G, bias, act)
    # the oracle rounds its double once to fp32: within half an fp32 ulp of the
    # value, plus the two doubles' rounding differences
    assert np.all(np.abs(y - ref) <= np.abs(ref) * 2.0 ** -24 * 1.001 + mag * 1e-13 + 1e-300)


@pytest.mark.parametrize("G", [1, 2, 16, 32, 128])
def test_quantizer_invariants(G):
    rng = np.random.default_rng(G)
    N, K = 20, 256
    W = (rng.standard_normal((N, K)) * np.exp(rng.uniform(-3, 3, (N, K // G))).repeat(G, axis=1)).astype(np.float32)
    W[3, :G] = 0.0                                   # an all-zero group
    Wq, sw = oracle.quantize_weights_kgroups(W, G)
    assert np.all(np.abs(Wq.astype(np.int32)) <= 127)
    assert sw[3, 0] == 0.0 and np.all(Wq[3, :G] == 0)
    Wb = W.reshape(N, K // G, G)
    qb = Wq.reshape(N, K // G, G).astype(np.int32)
    s = sw.astype(np.float64)[:, :, None]
    # rounding error at most half a step (plus the fp32 roundings of 127/absmax and v*inv)
    assert np.all(np.abs(Wb - qb * s) <= s * (0.5 + 2.0 ** -16) + 1e-30)
    # every non-zero group has a code of magnitude 127 where its absmax sits
    am = np.argmax(np.abs(Wb), axis=2)
    top = np.take_along_axis(qb, am[:, :, None], axis=2)[:, :, 0]
    nz = sw > 0
    assert np.all(np.abs(top[nz]) == 127)
    assert np.all(sw == (np.abs(Wb).max(axis=2) / np.float32(127)).astype(np.float32))


def test_kgroups_follow_input_channel_ranges():
    """Input channels whose ranges differ by two decades: per-row scales give
    the small channels few levels; K-axis groups give each its own range."""
    rng = np.random.default_rng(7)
    N, K, G = 64, 512, 32
    m = np.exp(rng.uniform(np.log(0.1), np.log(10.0), K // G)).repeat(G)
    W = (0.02 * rng.standard_normal((N, K)) * m[None, :]).astype(np.float32)
    Wq, sw = oracle.quantize_weights_kgroups(W, G)
    Wq1, s1 = oracle.quantize_weights(W, 1)
    err_k = np.linalg.norm(W - Wq * np.repeat(sw, G, axis=1)) / np.linalg.norm(W)
    err_r = np.linalg.norm(W - Wq1 * s1[:, None]) / np.linalg.norm(W)
    assert err_k < 0.5 * err_r
    # and the linear on random activations follows the float64 product more closely
    x = rng.standard_normal((32, K)).astype(np.float32)
    xq, st = oracle.quantize_rows(x)
    exact = x.astype(np.float64) @ W.astype(np.float64).T
    yk = oracle.linear_kgroups(xq, st, Wq, sw, G)
    yr = oracle.linear(xq, st, Wq1, s1, 1)
    assert np.linalg.norm(yk - exact) < np.linalg.norm(yr - exact)


def test_bad_arguments_are_refused():
    W = np.ones((4, 96), np.float32)
    with pytest.raises(oracle.OracleError):
        oracle.quantize_weights_kgroups(W, 64)       # 96 is not a multiple of 64
    Wq, sw = oracle.quantize_weights_kgroups(W, 32)
    with pytest.raises(oracle.OracleError):
        oracle.linear_kgroups(np.ones((2, 96), np.int8), np.ones(2, np.float32), Wq, sw, 16)


MUTANTS = ["row_groups", "scales_transposed", "last_group_dropped", "token_scale_on_each_group"]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_kgroup_pins_catch_planted_mistakes(mutant):
    """Each plausible mistake, planted on the CPU, changes the hand-worked
    codes, scales or outputs of the first golden block."""
    b = BLOCKS[0]
    W, G, xq, st, bias = _case(b)
    N, K = W.shape
    ng = K // G
    Wq, sw = oracle.quantize_weights_kgroups(W, G)
    if mutant == "row_groups":                       # groups of rows instead of columns
        Wq, s1 = oracle.quantize_weights(W, 1)
        sw = np.repeat(s1[:, None], ng, axis=1)
    elif mutant == "scales_transposed":              # s_w[j, o] read as s_w[o, j]
        sw = np.ascontiguousarray(sw.T).reshape(N, ng)
    elif mutant == "last_group_dropped":
        sw = sw.copy()
        sw[:, -1] = 0.0
    y = oracle.linear_kgroups(xq, st, Wq, sw, G, bias)
    if mutant == "token_scale_on_each_group":        # token scale applied per group, then summed with bias each time
        y = np.zeros_like(y)
        for j in range(ng):
            sl = slice(j * G, (j + 1) * G)
            y += oracle.linear_kgroups(xq[:, sl], st, Wq[:, sl], sw[:, j:j + 1], G, bias)
    ok = (np.array_equal(Wq, np.atleast_2d(b["Wq"]).astype(np.int8))
          and np.array_equal(sw, b["s_w"].astype(np.float32).reshape(N, ng))
          and np.array_equal(y, np.atleast_2d(b["y"]).astype(np.float32)))
    assert not ok
