"""The workloads at full size, in the launch configuration the benchmark
times, against the CPU oracle: every output where the oracle is quick, a
seeded sample of token rows otherwise (each oracle row depends only on that
row of the inputs, so sampled rows are checked exactly as full ones)."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import (BF16_TOL, F32_TOL, assert_codes_close, assert_dequant_close,
                               assert_scales_close, dequant_magnitude, dev, dev_act, host,
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


def test_tiny_linear_end_to_end(zq):
    """16 x 64 fp32 -> LN + quant -> W8A8 linear (G = 16) -> fp32, all outputs."""
    w = inputs.tiny()
    lin = w.layers[0]
    Wq, sg = zq.zq_quantize_weights(dev(lin.W), lin.group_rows)
    Wq_ref, sg_ref = oracle.quantize_weights(lin.W, lin.group_rows)
    np.testing.assert_array_equal(host(Wq), Wq_ref)
    np.testing.assert_array_equal(host(sg), sg_ref)
    x = dev_act(w.x)
    q, s = zq.zq_ln_quant(x, dev(w.gamma), dev(w.beta), w.eps)
    q_ref, s_ref = oracle.ln_quant(w.x.f32, w.gamma, w.beta, w.eps)
    assert_codes_close(host(q), q_ref, max_frac=1.0 / q_ref.size)   # at most one code of 1024
    assert_scales_close(host(s), s_ref)
    # the linear, fed the GPU's codes on both sides
    qh, sh = host(q), host(s)
    y = zq.zq_w8a8_linear(q, s, Wq, sg, lin.group_rows, bias=dev(lin.bias), out_kind=zq.ZQ_OUT_F32)
    acc = oracle.gemm_i32(qh, Wq_ref)
    assert_dequant_close(host(y), oracle.dequant(acc, sh, sg_ref, lin.group_rows, lin.bias),
                         dequant_magnitude(acc, sh, sg_ref, lin.group_rows, lin.bias), F32_TOL)
    # the one-call block gives the same output
    y2 = zq.zq_linear_block(x, dev(w.gamma), dev(w.beta), w.eps, Wq, sg, lin.group_rows,
                            bias=dev(lin.bias), out_kind=zq.ZQ_OUT_F32)
    assert torch.equal(y, y2)


def _quantized_layers(zq, w):
    out = []
    for lin in w.layers:
        Wq, sg = zq.zq_quantize_weights(dev(lin.W), lin.group_rows)
        out.append((Wq, sg, dev(lin.bias), lin))
    return out


def test_bert_ffn_block_stagewise(zq):
    """x bf16 [4096, 768] -> LN+quant -> W1 (+bias, GeLU, requant) -> W2 (+bias) -> bf16."""
    w = inputs.bert_ffn()
    (W1q, s1, b1, l1), (W2q, s2, b2, l2) = _quantized_layers(zq, w)
    x = dev_act(w.x)
    q1, st1 = zq.zq_ln_quant(x, dev(w.gamma), dev(w.beta), w.eps)
    q2, st2 = zq.zq_w8a8_linear(q1, st1, W1q, s1, 64, bias=b1, act=zq.ZQ_ACT_GELU,
                                out_kind=zq.ZQ_OUT_I8_REQUANT)
    y = zq.zq_w8a8_linear(q2, st2, W2q, s2, 64, bias=b2, out_kind=zq.ZQ_OUT_BF16)
    torch.cuda.synchronize()
    rows = sample_rows(w.x.f32.shape[0], 64, seed=1)
    W1_ref, s1_ref = oracle.quantize_weights(l1.W, 64)
    W2_ref, s2_ref = oracle.quantize_weights(l2.W, 64)
    # stage 1: LN + quant on all rows
    q1_ref, st1_ref = oracle.ln_quant(w.x.f32, w.gamma, w.beta, w.eps)
    assert_codes_close(host(q1), q1_ref)
    assert_scales_close(host(st1), st1_ref)
    # stage 2: W1 + GeLU + requant, fed the GPU's stage-1 codes
    q1h, st1h = host(q1)[rows], host(st1)[rows]
    q2_ref, st2_ref = oracle.linear_requant(q1h, st1h, W1_ref, s1_ref, 64, l1.bias, oracle.ACT_GELU)
    assert_codes_close(host(q2)[rows], q2_ref)
    assert_scales_close(host(st2)[rows], st2_ref)
    # stage 3: W2, fed the GPU's stage-2 codes
    q2h, st2h = host(q2)[rows], host(st2)[rows]
    acc = oracle.gemm_i32(q2h, W2_ref)
    assert_dequant_close(host(y)[rows], oracle.dequant(acc, st2h, s2_ref, 64, l2.bias),
                         dequant_magnitude(acc, st2h, s2_ref, 64, l2.bias), BF16_TOL)
    # end to end against the oracle's own pipeline: relative Frobenius error
    y_ref, _ = oracle.ffn_block(w.x.f32[rows], w.gamma, w.beta, w.eps, W1_ref, s1_ref, l1.bias,
                                W2_ref, s2_ref, l2.bias, 64)
    rel = np.linalg.norm(host(y)[rows] - y_ref) / np.linalg.norm(y_ref)
    assert rel <= 1e-2, rel


def test_gptj_qkv_full_size(zq):
    """x bf16 [2048, 4096] -> LN+quant -> W [12288, 4096] G=128 -> bf16."""
    w = inputs.gptj_qkv()
    ((Wq, sg, b, lin),) = _quantized_layers(zq, w)
    x = dev_act(w.x)
    q, st = zq.zq_ln_quant(x, dev(w.gamma), dev(w.beta), w.eps)
    y = zq.zq_w8a8_linear(q, st, Wq, sg, 128, bias=b, out_kind=zq.ZQ_OUT_BF16)
    acc_gpu = zq.zq_w8a8_linear(q, st, Wq, sg, 128, out_kind=zq.ZQ_OUT_I32_RAW)
    # full coverage of the accumulators against the library int8 matmul
    assert torch.equal(acc_gpu, torch._int_mm(q, Wq.t()))
    W_ref, sg_ref = oracle.quantize_weights(lin.W, 128)
    np.testing.assert_array_equal(host(Wq), W_ref)
    q_ref, st_ref = oracle.ln_quant(w.x.f32, w.gamma, w.beta, w.eps)
    assert_codes_close(host(q), q_ref)
    assert_scales_close(host(st), st_ref)
    rows = sample_rows(2048, 24, seed=2)
    qh, sth = host(q)[rows], host(st)[rows]
    acc = oracle.gemm_i32(qh, W_ref)
    np.testing.assert_array_equal(host(acc_gpu)[rows], acc)
    assert_dequant_close(host(y)[rows], oracle.dequant(acc, sth, sg_ref, 128, lin.bias),
                         dequant_magnitude(acc, sth, sg_ref, 128, lin.bias), BF16_TOL)


def test_neox_decode_full_size(zq):
    """x bf16 [16, 6144] -> token quant -> W [24576, 6144] G=256 + bias + GeLU -> bf16."""
    w = inputs.neox_decode()
    ((Wq, sg, b, lin),) = _quantized_layers(zq, w)
    x = dev_act(w.x)
    q, st = zq.zq_act_quant(x)
    y = zq.zq_w8a8_linear(q, st, Wq, sg, 256, bias=b, act=zq.ZQ_ACT_GELU, out_kind=zq.ZQ_OUT_BF16)
    acc_gpu = zq.zq_w8a8_linear(q, st, Wq, sg, 256, out_kind=zq.ZQ_OUT_I32_RAW)
    W_ref, sg_ref = oracle.quantize_weights(lin.W, 256)
    np.testing.assert_array_equal(host(Wq), W_ref)
    np.testing.assert_array_equal(host(sg), sg_ref)
    q_ref, st_ref = oracle.quantize_rows(w.x.f32)
    np.testing.assert_array_equal(host(q), q_ref)
    np.testing.assert_array_equal(host(st), st_ref)
    acc = oracle.gemm_i32(q_ref, W_ref)
    np.testing.assert_array_equal(host(acc_gpu), acc)
    y_ref = oracle.dequant(acc, st_ref, sg_ref, 256, lin.bias, oracle.ACT_GELU)
    assert_dequant_close(host(y), y_ref, dequant_magnitude(acc, st_ref, sg_ref, 256, lin.bias),
                         BF16_TOL)
    # the one-call block (token quant + linear) gives the same output
    y2 = zq.zq_linear_block(x, None, None, 0.0, Wq, sg, 256, bias=b, act=zq.ZQ_ACT_GELU,
                            out_kind=zq.ZQ_OUT_BF16)
    assert torch.equal(y, y2)


@pytest.mark.parametrize("M", inputs.GEMM_SWEEP_M)
def test_gemm_sweep_point(zq, M):
    """M x 8192 x 8192, G = 128, bf16 out: sampled rows against the oracle."""
    idx = inputs.GEMM_SWEEP_M.index(M)
    w = inputs.gemm_sweep_point(M, idx)
    ((Wq, sg, b, lin),) = _quantized_layers(zq, w)
    q, st = zq.zq_act_quant(dev_act(w.x))
    y = zq.zq_w8a8_linear(q, st, Wq, sg, 128, bias=b, out_kind=zq.ZQ_OUT_BF16)
    torch.cuda.synchronize()
    rows = sample_rows(M, 12, seed=idx)
    W_ref, sg_ref = oracle.quantize_weights(lin.W, 128)
    q_ref, st_ref = oracle.quantize_rows(w.x.f32[rows])
    np.testing.assert_array_equal(host(q)[rows], q_ref)
    np.testing.assert_array_equal(host(st)[rows], st_ref)
    acc = oracle.gemm_i32(q_ref, W_ref)
    assert_dequant_close(host(y)[rows], oracle.dequant(acc, st_ref, sg_ref, 128, lin.bias),
                         dequant_magnitude(acc, st_ref, sg_ref, 128, lin.bias), BF16_TOL)
