"""GPU parity of the SmoothQuant offline steps against the CPU oracle, through
the C ABI ("探秘Transformer系列之（36）— 大模型量化方案" §1.3;
"SmoothQuant技术解析：大模型INT8量化的突破与实践" §2.2, §3): per-channel
calibration absmax (raw or through the LayerNorm), the smoothing factors, the
fold into gamma/beta and the weights, and the smoothed W8A8 layer end to
end."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import assert_codes_close, assert_scales_close, dev, dev_act, host
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


def _acts(seed, T, H, dtype):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(4.0, size=(T, H)).astype(np.float32)
    ch = rng.permutation(H)[: max(1, H // 96)]
    x[:, ch] *= 30.0
    return inputs._as_act(x, dtype == "bf16")


CAL_SHAPES = [(1, 16, "f32"), (33, 64, "bf16"), (100, 768, "bf16"), (257, 1040, "f32"),
              (64, 4096, "bf16"), (5, 12288, "bf16"), (9000, 768, "bf16"), (40, 32768, "bf16"),
              (70, 2064, "f32")]


@pytest.mark.parametrize("T,H,dtype", CAL_SHAPES)
def test_calibrate_raw_bit_exact(zq, T, H, dtype):
    a = _acts(T + H, T, H, dtype)
    amax = zq.zq_smooth_calibrate(dev_act(a))
    np.testing.assert_array_equal(host(amax), oracle.channel_absmax(a.f32))


@pytest.mark.parametrize("T,H,dtype", CAL_SHAPES)
def test_calibrate_layernorm_running_max(zq, T, H, dtype):
    """Two batches accumulate into one running max; the activation is the
    LayerNorm output (fp32 on the GPU, fp64 in the oracle)."""
    a = _acts(3 * T + H, T, H, dtype)
    b = _acts(5 * T + H, T, H, dtype)
    rng = np.random.default_rng(H)
    gamma = (1 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(H)).astype(np.float32)
    g, bt = dev(gamma), dev(beta)
    amax = zq.zq_smooth_calibrate(dev_act(a), g, bt, 1e-5)
    amax = zq.zq_smooth_calibrate(dev_act(b), g, bt, 1e-5, amax=amax)
    ref = oracle.channel_absmax(oracle.layernorm(b.f32, gamma, beta, 1e-5),
                                oracle.channel_absmax(oracle.layernorm(a.f32, gamma, beta, 1e-5)))
    np.testing.assert_allclose(host(amax), ref, rtol=1e-5, atol=1e-6)


def test_calibrate_rejects_too_wide_rows(zq):
    x = torch.zeros((2, 32784), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(zq.ZQError):
        zq.zq_smooth_calibrate(x)


def test_calibrate_zero_channel_and_edge_rows(zq):
    a = _acts(11, 70, 48, "f32")
    x = a.f32.copy()
    x[:, 7] = 0.0
    amax = host(zq.zq_smooth_calibrate(dev(x)))
    assert amax[7] == 0.0
    np.testing.assert_array_equal(amax, np.abs(x).max(0))


@pytest.mark.parametrize("N,K,alpha", [(16, 16, 0.5), (48, 64, 0.5), (3072, 768, 0.5), (768, 3072, 0.8),
                                       (100, 96, 1.0), (100, 96, 0.0), (12288, 4096, 0.5)])
def test_smooth_weights_parity(zq, N, K, alpha):
    """Factors within one fp32 ulp of the oracle's (powers in double on both
    sides); given the GPU's factors the fold is bit-exact."""
    rng = np.random.default_rng(N + K)
    W = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    W[:, 3] *= 10.0
    amax = np.abs(rng.standard_t(3.0, size=K)).astype(np.float32) * 5
    amax[5] = 0.0                                  # a channel never active: s = 1
    gamma = (1 + 0.1 * rng.standard_normal(K)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(K)).astype(np.float32)
    Wo, go, bo, s = zq.zq_smooth_weights(dev(W), dev(amax), alpha, dev(gamma), dev(beta))
    s_h = host(s)
    s_ref = oracle.smooth_factors(amax, oracle.weight_col_absmax(W), alpha)
    np.testing.assert_allclose(s_h, s_ref, rtol=2 ** -23, atol=0)
    assert s_h[5] == 1.0
    Wo_ref, go_ref, bo_ref = oracle.smooth_fold(W, s_h, gamma, beta)
    np.testing.assert_array_equal(host(Wo), Wo_ref)
    np.testing.assert_array_equal(host(go), go_ref)
    np.testing.assert_array_equal(host(bo), bo_ref)


def test_smooth_weights_in_place(zq):
    rng = np.random.default_rng(3)
    W = (0.02 * rng.standard_normal((64, 128))).astype(np.float32)
    amax = np.abs(rng.standard_normal(128)).astype(np.float32) + 0.1
    gamma = np.ones(128, np.float32)
    Wd, gd = dev(W), dev(gamma)
    _, _, _, s = zq.zq_smooth_weights(Wd, dev(amax), 0.5, gd, None, W_out=Wd, gamma_out=gd)
    s_h = host(s)
    Wo_ref, go_ref, _ = oracle.smooth_fold(W, s_h, gamma)
    np.testing.assert_array_equal(host(Wd), Wo_ref)
    np.testing.assert_array_equal(host(gd), go_ref)


def test_smooth_weights_rejects_bad_alpha(zq):
    W = dev(np.ones((16, 16), np.float32))
    a = dev(np.ones(16, np.float32))
    with pytest.raises(zq.ZQError):
        zq.zq_smooth_weights(W, a, 1.5)


def test_smoothed_bert_w1_end_to_end(zq):
    """Calibrate on the GPU, fold, quantize the smoothed weights, then the
    unchanged online path (LN + quant, W8A8 linear): stage-wise parity with
    the oracle fed the GPU's factors, and the smoothed layer is closer to
    the float64 product than the unsmoothed one."""
    w = inputs.bert_ffn(T=512)
    lin = w.layers[0]
    G = lin.group_rows
    x = dev_act(w.x)
    g, b = dev(w.gamma), dev(w.beta)
    amax = zq.zq_smooth_calibrate(x, g, b, w.eps)
    Wo, go, bo, s = zq.zq_smooth_weights(dev(lin.W), amax, 0.5, g, b)
    Wq, sg = zq.zq_quantize_weights(Wo, G)
    q, st = zq.zq_ln_quant(x, go, bo, w.eps)
    y = host(zq.zq_w8a8_linear(q, st, Wq, sg, G, out_kind=zq.ZQ_OUT_F32))

    # oracle, fed the GPU's factors (the LN-calibrated maxima differ in fp32 rounding)
    s_h = host(s)
    Wo_ref, go_ref, bo_ref = oracle.smooth_fold(lin.W, s_h, w.gamma, w.beta)
    np.testing.assert_array_equal(host(Wo), Wo_ref)
    Wq_ref, sg_ref = oracle.quantize_weights(Wo_ref, G)
    np.testing.assert_array_equal(host(Wq), Wq_ref)
    q_ref, st_ref = oracle.ln_quant(w.x.f32, go_ref, bo_ref, w.eps)
    assert_codes_close(host(q), q_ref)
    assert_scales_close(host(st), st_ref)

    ref = (torch.nn.functional.layer_norm(torch.from_numpy(w.x.f32).double(), (w.x.f32.shape[1],),
                                          torch.from_numpy(w.gamma).double(),
                                          torch.from_numpy(w.beta).double(), eps=w.eps).numpy()
           @ lin.W.astype(np.float64).T)
    err_s = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    q0, st0 = zq.zq_ln_quant(x, g, b, w.eps)
    Wq0, sg0 = zq.zq_quantize_weights(dev(lin.W), G)
    y0 = host(zq.zq_w8a8_linear(q0, st0, Wq0, sg0, G, out_kind=zq.ZQ_OUT_F32))
    err_0 = np.linalg.norm(y0 - ref) / np.linalg.norm(ref)
    assert err_s < 0.8 * err_0
