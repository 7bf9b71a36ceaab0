"""GPU parity of the memory-bound quantizers against the CPU oracle, through
the C ABI: weight group quantization, fused LayerNorm + token quantization,
fused (bias +) GeLU + token quantization."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import (assert_codes_close, assert_scales_close, dev, dev_act, host,
                               sample_rows)
from w8a8_post_quantized_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def zq():
    from w8a8_post_quantized_b200 import zq as m
    m.lib()
    return m


@pytest.fixture(autouse=True)
def _device_status_clean(zq):
    yield
    zq.zq_device_status()


def _rows(seed, T, H, dtype, outliers=True, t_nu=3.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(t_nu, size=(T, H)).astype(np.float32)
    if outliers and H >= 32:
        ch = rng.permutation(H)[: max(1, H // 128)]
        x[:, ch] *= 30.0
    return inputs._as_act(x, dtype == "bf16")


ROW_SHAPES = [
    (16, 64, "f32"), (1, 16, "bf16"), (7, 48, "bf16"), (33, 768, "bf16"), (129, 1024, "f32"),
    (5, 4096, "bf16"), (3, 6144, "bf16"), (2, 12288, "bf16"), (1, 65536, "bf16"),
    (300, 2064, "bf16"), (1000, 512, "f32"), (9, 12288, "f32"),
    (3, 32768, "bf16"),      # longest row of the pipelined kernel (bf16)
    (2, 40960, "bf16"),      # beyond it: the register kernel
    (5, 16384, "f32"),       # longest fp32 row of the pipelined kernel
    (4097, 768, "bf16"),     # partial last stage
]


@pytest.mark.parametrize("T,H,dtype", ROW_SHAPES)
def test_act_quant_bit_exact(zq, T, H, dtype):
    a = _rows(T * 1000 + H, T, H, dtype)
    q, s = zq.zq_act_quant(dev_act(a))
    q_ref, s_ref = oracle.quantize_rows(a.f32)
    np.testing.assert_array_equal(host(q), q_ref)
    np.testing.assert_array_equal(host(s), s_ref)


@pytest.mark.parametrize("T,H,dtype", [(16, 64, "f32"), (37, 768, "bf16"), (4, 6144, "bf16")])
def test_act_quant_with_bias_bit_exact(zq, T, H, dtype):
    a = _rows(7 + T, T, H, dtype)
    bias = (0.01 * np.random.default_rng(T).standard_normal(H)).astype(np.float32)
    q, s = zq.zq_act_quant(dev_act(a), bias=dev(bias))
    q_ref, s_ref = oracle.act_quant(a.f32, bias, oracle.ACT_NONE)
    np.testing.assert_array_equal(host(q), q_ref)
    np.testing.assert_array_equal(host(s), s_ref)


@pytest.mark.parametrize("T,H,dtype", [(16, 64, "f32"), (64, 3072, "bf16"), (16, 6144, "bf16"),
                                       (3, 12288, "bf16")])
def test_act_quant_gelu(zq, T, H, dtype):
    a = _rows(11 + H, T, H, dtype)
    bias = (0.01 * np.random.default_rng(H).standard_normal(H)).astype(np.float32)
    q, s = zq.zq_act_quant(dev_act(a), bias=dev(bias), act=zq.ZQ_ACT_GELU)
    q_ref, s_ref = oracle.act_quant(a.f32, bias, oracle.ACT_GELU)
    assert_codes_close(host(q), q_ref)
    assert_scales_close(host(s), s_ref)


def test_act_quant_zero_rows(zq):
    x = np.zeros((5, 256), np.float32)
    x[2, 7] = -3.0
    q, s = zq.zq_act_quant(dev(x))
    q, s = host(q), host(s)
    assert s[0] == 0 and s[1] == 0 and not q[[0, 1, 3, 4]].any()
    assert q[2, 7] == -127 and s[2] == np.float32(3.0) / np.float32(127.0)


@pytest.mark.parametrize("T,H,dtype", ROW_SHAPES)
def test_ln_quant_parity(zq, T, H, dtype):
    a = _rows(T * 7 + H, T, H, dtype)
    rng = np.random.default_rng(H)
    gamma = (1.0 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(H)).astype(np.float32)
    q, s = zq.zq_ln_quant(dev_act(a), dev(gamma), dev(beta), 1e-5)
    q_ref, s_ref = oracle.ln_quant(a.f32, gamma, beta, 1e-5)
    assert_codes_close(host(q), q_ref)
    assert_scales_close(host(s), s_ref)


def test_ln_quant_special_rows(zq):
    H = 128
    g = np.ones(H, np.float32)
    b = np.zeros(H, np.float32)
    x = np.zeros((3, H), np.float32)
    x[0] = 5.0                                     # constant row, beta = 0 -> all zero
    x[1] = np.tile([2.0, -2.0], H // 2)            # [a, -a] -> +-127
    x[2] = np.arange(H, dtype=np.float32)
    q, s = zq.zq_ln_quant(dev(x), dev(g), dev(b), 1e-5)
    q, s = host(q), host(s)
    assert s[0] == 0 and not q[0].any()
    np.testing.assert_array_equal(q[1], np.tile([127, -127], H // 2))
    q_ref, s_ref = oracle.ln_quant(x[2:], g, b, 1e-5)
    assert_codes_close(q[2:], q_ref)


def test_ln_quant_bert_full_size(zq):
    w = inputs.bert_ffn()
    q, s = zq.zq_ln_quant(dev_act(w.x), dev(w.gamma), dev(w.beta), w.eps)
    q_ref, s_ref = oracle.ln_quant(w.x.f32, w.gamma, w.beta, w.eps)
    assert_codes_close(host(q), q_ref)
    assert_scales_close(host(s), s_ref)


@pytest.mark.parametrize("T,H", [(1024, 12288), (65536, 1024), (16384, 4096), (64, 4096), (1, 1024)])
def test_ln_quant_sweep_points(zq, T, H):
    idx = inputs.LN_SWEEP_T.index(T) * len(inputs.LN_SWEEP_H) + inputs.LN_SWEEP_H.index(H)
    w = inputs.ln_sweep_point(T, H, idx)
    q, s = zq.zq_ln_quant(dev_act(w.x), dev(w.gamma), dev(w.beta), w.eps)
    rows = sample_rows(T, 64, seed=idx)
    q_ref, s_ref = oracle.ln_quant(w.x.f32[rows], w.gamma, w.beta, w.eps)
    assert_codes_close(host(q)[rows], q_ref)
    assert_scales_close(host(s)[rows], s_ref)


WEIGHT_CASES = [
    ("tiny", lambda: inputs.tiny().layers[0]),
    ("bert_w1", lambda: inputs.bert_ffn().layers[0]),
    ("bert_w2", lambda: inputs.bert_ffn().layers[1]),
    ("gptj", lambda: inputs.gptj_qkv().layers[0]),
    ("neox", lambda: inputs.neox_decode().layers[0]),
]


@pytest.mark.parametrize("name,make", WEIGHT_CASES, ids=[c[0] for c in WEIGHT_CASES])
def test_quantize_weights_bit_exact(zq, name, make):
    lin = make()
    Wq, s = zq.zq_quantize_weights(dev(lin.W), lin.group_rows)
    Wq_ref, s_ref = oracle.quantize_weights(lin.W, lin.group_rows)
    np.testing.assert_array_equal(host(s), s_ref)
    np.testing.assert_array_equal(host(Wq), Wq_ref)


@pytest.mark.parametrize("N,K,G", [(16, 16, 16), (48, 64, 1), (64, 48, 64), (272, 80, 16)])
def test_quantize_weights_edge_groups(zq, N, K, G):
    rng = np.random.default_rng(N + K + G)
    W = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    W[:G] = 0.0                                   # an all-zero group
    Wq, s = zq.zq_quantize_weights(dev(W), G)
    Wq_ref, s_ref = oracle.quantize_weights(W, G)
    np.testing.assert_array_equal(host(s), s_ref)
    np.testing.assert_array_equal(host(Wq), Wq_ref)
    assert host(s)[0] == 0.0
