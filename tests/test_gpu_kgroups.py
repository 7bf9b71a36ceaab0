"""GPU parity of the K-axis weight groups against the CPU oracle, through the
C ABI (group-wise weights of "[2022 NeurIPS] ZeroQuant: Efficient and
Affordable Post-Training Quantization for Large-Scale Transformers" and
"探秘Transformer系列之（36）— 大模型量化方案" §1.2.2 read along the input axis,
reading R17 of the oracle).

The quantizer is compared bit for bit (codes and scales).  The linear is fed
the oracle's codes and scales, so the only difference left is fp32
arithmetic: the kernel sums the groups' scaled partial products in fp32
(one rounding per group) where the oracle sums in double, so the bound is
|y - ref| <= tol * (s_tok * sum_j |s_w acc_j| + |bias|) with
tol = max(1e-5, (groups + 2) * 2^-24) for fp32 output and 1e-2 for bf16.
Shapes cover groups smaller than a 128-byte stage (several groups per
stage), groups of several stages, a group size that is not a power of two
(groups straddle stages), ragged T and N, one token, and the full GPT-J QKV
projection on sampled rows."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import BF16_TOL, F32_TOL, assert_codes_close, dev, dev_act, host, sample_rows
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


def _weights(N, K, G, seed):
    """Weights whose input-channel blocks differ in range (the case K-axis
    groups exist for), with one all-zero group."""
    rng = np.random.default_rng(seed)
    m = np.exp(rng.uniform(np.log(0.1), np.log(10.0), size=(1, K // 16))).repeat(16, axis=1)
    W = (0.02 * rng.standard_normal((N, K)) * m).astype(np.float32)
    W[N // 2, :G] = 0.0
    return W


@pytest.mark.parametrize("N,K,G", [(96, 256, 32), (300, 768, 128), (1000, 1024, 64), (64, 4096, 256),
                                   (7, 96, 96), (33, 48, 16), (16, 64, 1), (128, 12288, 4096)])
def test_quantizer_bit_exact(zq, N, K, G):
    W = _weights(N, K, G, N + K + G)
    Wq, sw = zq.zq_quantize_weights_kgroups(dev(W), G)
    Wq_ref, sw_ref = oracle.quantize_weights_kgroups(W, G)
    np.testing.assert_array_equal(host(Wq), Wq_ref)
    assert tuple(sw.shape) == (K // G, N)
    np.testing.assert_array_equal(host(sw), sw_ref.T)


def _linear_case(T, K, N, G, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(4.0, size=(T, K)).astype(np.float32)
    x[:, rng.permutation(K)[: max(1, K // 100)]] *= 25.0
    xq, st = oracle.quantize_rows(x)
    W = _weights(N, K, G, seed + 1)
    Wq, sw = oracle.quantize_weights_kgroups(W, G)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    return xq, st, Wq, sw, bias


def _magnitude(xq, st, Wq, sw, G, bias):
    """s_tok[t] * sum_j |s_w[o, j] acc_j[t, o]| + |bias[o]| in float64 (exact
    integer partial products: |acc_j| < 2^53)."""
    T, K = xq.shape
    mag = np.zeros((T, Wq.shape[0]))
    for j in range(K // G):
        blk = slice(j * G, (j + 1) * G)
        acc = xq[:, blk].astype(np.float64) @ Wq[:, blk].astype(np.float64).T
        mag += np.abs(acc) * np.abs(sw[:, j].astype(np.float64))[None, :]
    return mag * np.abs(st.astype(np.float64))[:, None] + np.abs(bias.astype(np.float64))[None, :]


def _tol(K, G, out):
    return max(F32_TOL, (K // G + 2) * 2.0 ** -24) if out == "f32" else BF16_TOL


def _check(y, ref, mag, tol):
    err = np.abs(y.astype(np.float64) - ref.astype(np.float64))
    bad = err > tol * mag + 1e-30
    assert not bad.any(), f"{bad.sum()} outputs outside tolerance; worst {(err / (mag + 1e-30)).max():.3e}"


LINEAR_SHAPES = [
    (1, 32, 16, 32, 0, "f32"),        # one token, one k-step, a 16-column tile
    (16, 256, 128, 32, 0, "f32"),     # four groups per 128-byte stage
    (130, 384, 272, 64, 1, "f32"),    # two groups per stage; ragged T and N
    (64, 192, 48, 96, 0, "f32"),      # 96-column groups straddle stages
    (300, 768, 528, 128, 0, "bf16"),  # one group per stage
    (257, 1024, 384, 256, 1, "bf16"),  # a group spans two stages
    (1000, 4096, 1536, 128, 0, "f32"),  # several waves of tiles, 32 groups
    (513, 2048, 640, 32, 1, "f32"),   # 64 groups, the fp32-sum bound above 1e-5
    (192, 8192, 256, 64, 0, "f32"),   # 128 groups
    (64, 12288, 256, 256, 1, "bf16"),  # K = 12288: 48 groups of two stages
]


@pytest.mark.parametrize("T,K,N,G,act,out", LINEAR_SHAPES)
def test_linear_kgroups_matches_oracle(zq, T, K, N, G, act, out):
    xq, st, Wq, sw, bias = _linear_case(T, K, N, G, T + K + N + G)
    ok = zq.ZQ_OUT_F32 if out == "f32" else zq.ZQ_OUT_BF16
    y = zq.zq_w8a8_linear_kgroups(dev(xq), dev(st), dev(Wq), dev(np.ascontiguousarray(sw.T)), G, bias=dev(bias),
                                  act=act, out_kind=ok)
    ref = oracle.linear_kgroups(xq, st, Wq, sw, G, bias, act)
    _check(host(y), ref, _magnitude(xq, st, Wq, sw, G, bias), _tol(K, G, out))


def test_linear_kgroups_without_bias_and_repeated_calls(zq):
    """No bias; the same buffers twice (the accumulator slots are re-armed
    at every group, so a second launch sees the same state)."""
    T, K, N, G = 200, 512, 256, 64
    xq, st, Wq, sw, _ = _linear_case(T, K, N, G, 5)
    args = (dev(xq), dev(st), dev(Wq), dev(np.ascontiguousarray(sw.T)), G)
    y1 = zq.zq_w8a8_linear_kgroups(*args, out_kind=zq.ZQ_OUT_F32)
    y2 = zq.zq_w8a8_linear_kgroups(*args, out_kind=zq.ZQ_OUT_F32)
    assert torch.equal(y1, y2)
    zero = np.zeros(N, np.float32)
    ref = oracle.linear_kgroups(xq, st, Wq, sw, G)
    _check(host(y1), ref, _magnitude(xq, st, Wq, sw, G, zero), _tol(K, G, "f32"))


def test_linear_kgroups_zero_token_rows_give_the_bias(zq):
    """Rows whose codes and token scale are all zero (an all-zero input row)
    come out as exactly the bias; the other rows are unaffected."""
    T, K, N, G = 160, 512, 272, 128
    xq, st, Wq, sw, bias = _linear_case(T, K, N, G, 21)
    zero_rows = [0, 77, 159]
    xq[zero_rows] = 0
    st[zero_rows] = 0.0
    y = host(zq.zq_w8a8_linear_kgroups(dev(xq), dev(st), dev(Wq), dev(np.ascontiguousarray(sw.T)), G,
                                       bias=dev(bias), out_kind=zq.ZQ_OUT_F32))
    np.testing.assert_array_equal(y[zero_rows], np.broadcast_to(bias, (len(zero_rows), N)))
    ref = oracle.linear_kgroups(xq, st, Wq, sw, G, bias)
    _check(y, ref, _magnitude(xq, st, Wq, sw, G, bias), _tol(K, G, "f32"))


def test_gptj_qkv_kgroups_sampled_rows(zq):
    """The benchmark's projection at full size (2048 tokens, 4096 -> 12288,
    128-column groups, bf16 out), in the benchmark's launch configuration,
    checked on sampled rows."""
    T, K, N, G = 2048, 4096, 12288, 128
    rng = np.random.default_rng(3)
    x = (0.5 * rng.standard_t(4.0, size=(T, K))).astype(np.float32)
    xq, st = oracle.quantize_rows(x)
    W = _weights(N, K, G, 4)
    Wq_d, sw_d = zq.zq_quantize_weights_kgroups(dev(W), G)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    y = host(zq.zq_w8a8_linear_kgroups(dev(xq), dev(st), Wq_d, sw_d, G, bias=dev(bias), out_kind=zq.ZQ_OUT_BF16))
    rows = sample_rows(T, 24, seed=3)
    Wq, sw = host(Wq_d), np.ascontiguousarray(host(sw_d).T)
    Wq_ref, sw_ref = oracle.quantize_weights_kgroups(W, G)
    np.testing.assert_array_equal(Wq, Wq_ref)
    np.testing.assert_array_equal(sw, sw_ref)
    ref = oracle.linear_kgroups(xq[rows], st[rows], Wq, sw, G, bias)
    _check(y[rows], ref, _magnitude(xq[rows], st[rows], Wq, sw, G, bias), BF16_TOL)


def test_ln_quant_then_kgroup_linear(zq):
    """LayerNorm + token quantization on the GPU feeding the K-group linear:
    stage-wise the GEMM sees the GPU's own codes (then the bound above
    holds); end to end the output is within 1e-2 (relative Frobenius) of the
    oracle's composition, and closer to the float64 product than per-row
    weight scales on weights whose input channels differ in range."""
    w = inputs.bert_ffn(T=512)
    lin = w.layers[0]
    N, K = lin.W.shape
    G = 128
    W = lin.W * np.exp(np.random.default_rng(9).uniform(np.log(0.1), np.log(10.0), (1, K // G))).repeat(G, axis=1)
    W = W.astype(np.float32)
    q, st = zq.zq_ln_quant(dev_act(w.x), dev(w.gamma), dev(w.beta), w.eps)
    Wq_d, sw_d = zq.zq_quantize_weights_kgroups(dev(W), G)
    y = host(zq.zq_w8a8_linear_kgroups(q, st, Wq_d, sw_d, G, bias=dev(lin.bias), out_kind=zq.ZQ_OUT_F32))
    qh, sth = host(q), host(st)
    q_ref, st_ref = oracle.ln_quant(w.x.f32, w.gamma, w.beta, w.eps)
    assert_codes_close(qh, q_ref)
    Wq, sw = oracle.quantize_weights_kgroups(W, G)
    ref_stage = oracle.linear_kgroups(qh, sth, Wq, sw, G, lin.bias)
    _check(y, ref_stage, _magnitude(qh, sth, Wq, sw, G, lin.bias), _tol(K, G, "f32"))
    ref = oracle.ln_linear_kgroups(w.x.f32, w.gamma, w.beta, w.eps, Wq, sw, G, lin.bias)
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 1e-2
    a = oracle.layernorm(w.x.f32, w.gamma, w.beta, w.eps).astype(np.float64)
    exact = a @ W.astype(np.float64).T + lin.bias
    Wq1, s1 = zq.zq_quantize_weights(dev(W), 1)
    y1 = host(zq.zq_w8a8_linear(q, st, Wq1, s1, 1, bias=dev(lin.bias), out_kind=zq.ZQ_OUT_F32))
    assert np.linalg.norm(y - exact) < np.linalg.norm(y1 - exact)


def test_linear_kgroups_refuses_bad_arguments(zq):
    T, K, N = 64, 256, 128
    xq = torch.zeros((T, K), dtype=torch.int8, device="cuda")
    st = torch.ones(T, dtype=torch.float32, device="cuda")
    Wq = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    for G, sw_rows, out in [(16, K // 16, zq.ZQ_OUT_F32),    # group narrower than a k-step
                            (512, 1, zq.ZQ_OUT_F32),          # above 256 columns
                            (96, 3, zq.ZQ_OUT_F32),           # K % G != 0
                            (64, K // 64, zq.ZQ_OUT_I8_REQUANT)]:  # output kind not offered
        sw = torch.ones((sw_rows, N), dtype=torch.float32, device="cuda")
        with pytest.raises(zq.ZQError):
            zq.zq_w8a8_linear_kgroups(xq, st, Wq, sw, G, out_kind=out)
    sw = torch.ones(K // 64 * N + 1, dtype=torch.float32, device="cuda")[1:].view(K // 64, N)
    with pytest.raises(zq.ZQError):                               # scales not 16-byte aligned
        zq.zq_w8a8_linear_kgroups(xq, st, Wq, sw, 64, out_kind=zq.ZQ_OUT_F32)
    with pytest.raises(zq.ZQError):                               # N % 16 != 0
        zq.zq_w8a8_linear_kgroups(xq, st, Wq[:120], torch.ones((4, 120), device="cuda"), 64,
                                  out_kind=zq.ZQ_OUT_F32)
