"""GPU parity of the LLM.int8() mixed-precision decomposition against the CPU
oracle, through the C ABI ("探秘Transformer系列之（36）— 大模型量化方案" §1.1,
reading R16 of the oracle): outlier column selection with the masked
LayerNorm parameters, the fp16 outlier operands, the W8A8 linear with the
outlier product in its epilogue, and the whole decomposed layer."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import (BF16_TOL, F32_TOL, assert_codes_close, assert_dequant_close,
                               assert_scales_close, dev, dev_act, host)
from w8a8_post_quantized_b200 import inputs

pytestmark = pytest.mark.gpu
MAXO = 8


@pytest.fixture(scope="module")
def zq():
    from w8a8_post_quantized_b200 import zq as m
    m.lib()
    return m


@pytest.fixture(autouse=True)
def _device_status_clean(zq):
    yield
    zq.zq_device_status()


@pytest.mark.parametrize("K,n_out", [(16, 0), (64, 3), (768, 8), (768, 12), (12288, 5), (4096, 40)])
def test_select_matches_oracle(zq, K, n_out):
    rng = np.random.default_rng(K + n_out)
    amax = (rng.uniform(0, 5.9, K)).astype(np.float32)
    cols = rng.permutation(K)[:n_out]
    amax[cols] = rng.uniform(6.0, 50.0, n_out).astype(np.float32)
    if n_out:
        amax[cols[0]] = 6.0                          # the boundary value counts
    gamma = (1 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(K)).astype(np.float32)
    idx, count, gm, bm = zq.zq_llmint8_select(dev(amax), dev(gamma), dev(beta), 6.0)
    idx_ref, n_ref = oracle.outlier_columns(amax, 6.0, MAXO)
    assert int(host(count)[0]) == n_ref
    got = host(idx)
    np.testing.assert_array_equal(got[:idx_ref.size], idx_ref)
    assert np.all(got[idx_ref.size:] == -1)
    g_ref, b_ref = gamma.copy(), beta.copy()
    g_ref[idx_ref] = 0.0
    b_ref[idx_ref] = 0.0
    np.testing.assert_array_equal(host(gm), g_ref)
    np.testing.assert_array_equal(host(bm), b_ref)


def _layer(seed, T, K, N, G, dtype="bf16", scale=40.0, n_out=4):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, K)).astype(np.float32)
    x[:, rng.permutation(K)[:n_out]] *= scale
    xa = inputs._as_act(x, dtype == "bf16")
    gamma = (1 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(K)).astype(np.float32)
    W = (0.03 * rng.standard_normal((N, K))).astype(np.float32)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    return xa, gamma, beta, W, bias


def _gpu_parts(zq, xa, gamma, beta, W, eps=1e-5):
    x = dev_act(xa)
    g, b = dev(gamma), dev(beta)
    amax = zq.zq_smooth_calibrate(x, g, b, eps)
    idx, count, gm, bm = zq.zq_llmint8_select(amax, g, b, 6.0)
    q, st = zq.zq_ln_quant(x, gm, bm, eps)
    xo = zq.zq_llmint8_outlier_act(x, g, b, eps, idx, count)
    wo = zq.zq_llmint8_outlier_weights(dev(W), idx, count)
    return x, amax, idx, count, q, st, xo, wo


@pytest.mark.parametrize("T,K,N,dtype", [(64, 128, 96, "f32"), (300, 768, 512, "bf16"), (1000, 1024, 384, "bf16")])
def test_outlier_operands(zq, T, K, N, dtype):
    xa, gamma, beta, W, _ = _layer(T + K, T, K, N, 16, dtype)
    _, _, idx, count, _, _, xo, wo = _gpu_parts(zq, xa, gamma, beta, W)
    n = min(int(host(count)[0]), MAXO)
    ix = host(idx)[:n]
    assert n >= 1
    # weights: fp16 of the fp32 columns, round to nearest even, zeros past the count
    wo_h = host(wo.view(torch.int16)).view(np.float16)
    np.testing.assert_array_equal(wo_h[:, :n], W[:, ix].astype(np.float16))
    assert np.all(wo_h[:, n:] == 0)
    # activations: fp16 of the LayerNorm output (fp32 on the GPU, fp64 in the
    # oracle), so at most one fp16 ulp apart
    a = oracle.layernorm(xa.f32, gamma, beta, 1e-5)
    xo_h = host(xo.view(torch.int16)).view(np.float16).astype(np.float64)
    ref = a[:, ix].astype(np.float16).astype(np.float64)
    ulp = np.abs(ref) * 2.0 ** -10 + 2.0 ** -24
    assert np.all(np.abs(xo_h[:, :n] - ref) <= ulp)
    assert np.all(xo_h[:, n:] == 0)


@pytest.mark.parametrize("T,K,N,G,act,out", [(64, 128, 96, 16, 0, "f32"), (300, 768, 512, 64, 1, "f32"),
                                             (1000, 1024, 384, 128, 0, "bf16"), (130, 768, 3072, 64, 1, "bf16")])
def test_linear_llmint8_stagewise(zq, T, K, N, G, act, out):
    """The GEMM with the outlier epilogue, fed the GPU's codes and fp16
    operands on both sides: y = act(s_tok s_grp acc + xo wo^T + bias)."""
    xa, gamma, beta, W, bias = _layer(3 * T + K, T, K, N, G)
    _, _, idx, count, q, st, xo, wo = _gpu_parts(zq, xa, gamma, beta, W)
    Wq, sg = zq.zq_quantize_weights(dev(W), G)
    ok = zq.ZQ_OUT_F32 if out == "f32" else zq.ZQ_OUT_BF16
    y = zq.zq_w8a8_linear_llmint8(q, st, Wq, sg, G, xo, wo, bias=dev(bias), act=act, out_kind=ok)
    qh, sth, Wqh, sgh = host(q), host(st), host(Wq), host(sg)
    xo64 = host(xo.view(torch.int16)).view(np.float16).astype(np.float64)
    wo64 = host(wo.view(torch.int16)).view(np.float16).astype(np.float64)
    add = xo64 @ wo64.T
    acc = oracle.gemm_i32(qh, Wqh)
    ref = oracle.dequant_add(acc, sth, sgh, G, add, bias, act)
    mag = (np.abs(acc.astype(np.float64)) * sth[:, None].astype(np.float64)
           * np.repeat(sgh.astype(np.float64), G)[None, :] + np.abs(xo64) @ np.abs(wo64).T + np.abs(bias))
    assert_dequant_close(host(y).astype(np.float32), ref, mag, F32_TOL if out == "f32" else BF16_TOL)


def test_linear_llmint8_without_outliers_is_the_plain_linear(zq):
    xa, gamma, beta, W, bias = _layer(5, 200, 512, 640, 64, scale=1.0, n_out=0)
    x = dev_act(xa)
    q, st = zq.zq_ln_quant(x, dev(gamma), dev(beta), 1e-5)
    Wq, sg = zq.zq_quantize_weights(dev(W), 64)
    zeros_x = torch.zeros((200, MAXO), dtype=torch.float16, device="cuda")
    zeros_w = torch.zeros((640, MAXO), dtype=torch.float16, device="cuda")
    for ok in (zq.ZQ_OUT_F32, zq.ZQ_OUT_BF16):
        for act in (0, 1):
            y1 = zq.zq_w8a8_linear_llmint8(q, st, Wq, sg, 64, zeros_x, zeros_w, bias=dev(bias), act=act, out_kind=ok)
            y0 = zq.zq_w8a8_linear(q, st, Wq, sg, 64, bias=dev(bias), act=act, out_kind=ok)
            assert torch.equal(y0, y1)


def test_decomposed_layer_end_to_end(zq):
    """The whole decomposed layer on the GPU against the oracle's
    composition: the same outlier columns; outputs within 1e-2 relative
    (Frobenius); and, as the method promises, closer to the float64 product
    than the plain W8A8 layer."""
    w = inputs.bert_ffn(T=512)
    lin = w.layers[0]
    G = lin.group_rows
    x, amax, idx, count, q, st, xo, wo = _gpu_parts(zq, w.x, w.gamma, w.beta, lin.W, w.eps)
    Wq, sg = zq.zq_quantize_weights(dev(lin.W), G)
    y = host(zq.zq_w8a8_linear_llmint8(q, st, Wq, sg, G, xo, wo, bias=dev(lin.bias), act=0,
                                       out_kind=zq.ZQ_OUT_F32)).astype(np.float64)
    Wq_ref, sg_ref = oracle.quantize_weights(lin.W, G)
    y_ref, idx_ref, n_ref = oracle.int8_decomposed_ln_linear(w.x.f32, w.gamma, w.beta, w.eps, lin.W, Wq_ref,
                                                             sg_ref, G, lin.bias)
    assert int(host(count)[0]) == n_ref and n_ref >= 1
    np.testing.assert_array_equal(host(idx)[:idx_ref.size], idx_ref)
    assert np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref) < 1e-2
    a = oracle.layernorm(w.x.f32, w.gamma, w.beta, w.eps).astype(np.float64)
    exact = a @ lin.W.astype(np.float64).T + lin.bias
    q0, st0 = zq.zq_ln_quant(x, dev(w.gamma), dev(w.beta), w.eps)
    y0 = host(zq.zq_w8a8_linear(q0, st0, Wq, sg, G, bias=dev(lin.bias), out_kind=zq.ZQ_OUT_F32))
    assert np.linalg.norm(y - exact) < 0.8 * np.linalg.norm(y0 - exact)
