"""Parity of the requantizing linear (ZQ_OUT_I8_REQUANT) on the shapes the
thread-block-cluster kernel does not take -- output rows wider than 4096
features, and at most 64 tokens -- against the CPU oracle.

The per-token requantization follows "探秘Transformer系列之（36）— 大模型量化方案"
§1.2.2 (one dynamic scale per token, taken over the whole output row of the
linear, fused with the op that produces it) and the fused
"GEMM + DeQuantize" kernel of "[2022 NeurIPS] ZeroQuant: Efficient and
Affordable Post-Training Quantization for Large-Scale Transformers".  Every
output row is compared where the oracle is quick; the GPT-J FFN-up shape
(2048 x 4096 -> 16384) compares every row of the last 128-row block and a
seeded sample of the others (each oracle row depends only on that row of
the inputs)."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import assert_codes_close, assert_scales_close, dev, host, sample_rows

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


def _case(T, K, N, G, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(4.0, size=(T, K)).astype(np.float32)
    x[:, rng.permutation(K)[: max(1, K // 100)]] *= 25.0
    W = (0.02 * rng.standard_normal((N, K))
         * np.exp(rng.uniform(-1, 1, size=(N, 1)))).astype(np.float32)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    xq, s_tok = oracle.quantize_rows(x)
    Wq, s_grp = oracle.quantize_weights(W, G)
    return xq, s_tok, Wq, s_grp, bias


# (T, K, N, G): every case has N > 4096 or T <= 64
WIDE_SHAPES = [
    (65, 256, 4112, 16),      # first non-swapped T; N = 16 * 257 (a half-filled last 32-column chunk)
    (300, 384, 4608, 64),     # ragged T, N = 18 column tiles of 256
    (300, 256, 5120, 128),    # N = 20 column tiles
    (200, 320, 4160, 64),     # ragged T and a 64-column last tile; K not a multiple of 128
    (1000, 512, 8192, 64),    # 8 row blocks x 32 column tiles
    (16, 768, 6144, 64),      # decode-sized: swapped operand roles, 16 tokens
    (33, 1024, 4096, 64),     # swapped, 33 tokens
    (64, 512, 8192, 128),     # swapped, 64 tokens, wide
    (130, 64, 38144, 16),     # 149 column tiles per row: more than the SMs, the scratch route
]


def _ids(shapes):
    return [f"T{t}_K{k}_N{n}_G{g}" for t, k, n, g in shapes]


@pytest.mark.parametrize("T,K,N,G", WIDE_SHAPES, ids=_ids(WIDE_SHAPES))
@pytest.mark.parametrize("act", [0, 1], ids=["none", "gelu"])
def test_requant_wide_rows(zq, T, K, N, G, act):
    xq, s_tok, Wq, s_grp, bias = _case(T, K, N, G, seed=11 * T + N + act)
    q, s = zq.zq_w8a8_linear(dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G, bias=dev(bias), act=act,
                             out_kind=zq.ZQ_OUT_I8_REQUANT)
    q_ref, s_ref = oracle.linear_requant(xq, s_tok, Wq, s_grp, G, bias, act)
    qh = host(q)
    assert_codes_close(qh, q_ref)
    assert_scales_close(host(s), s_ref)
    assert np.all(np.abs(qh).max(axis=1) == 127)


def test_requant_gptj_ffn_up_sampled_rows(zq):
    """GPT-J-6B FFN-up shape (2048 tokens, 4096 -> 16384, 128-row groups,
    GeLU): every row of the last 128-row block plus a seeded sample."""
    T, K, N, G = 2048, 4096, 16384, 128
    xq, s_tok, Wq, s_grp, bias = _case(T, K, N, G, seed=2048)
    q, s = zq.zq_w8a8_linear(dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G, bias=dev(bias),
                             act=zq.ZQ_ACT_GELU, out_kind=zq.ZQ_OUT_I8_REQUANT)
    qh, sh = host(q), host(s)
    rows = np.unique(np.concatenate([np.arange(T - 128, T), sample_rows(T, 40, seed=7)]))
    q_ref, s_ref = oracle.linear_requant(xq[rows], s_tok[rows], Wq, s_grp, G, bias, oracle.ACT_GELU)
    assert_codes_close(qh[rows], q_ref)
    assert_scales_close(sh[rows], s_ref)
    assert np.all(np.abs(qh).max(axis=1) == 127)


def test_requant_workspace_is_small_when_fused(zq):
    """More than 64 tokens and at most one column tile per SM: the fused
    kernels need a word per row and per 128-row block, not the fp32 output;
    a call given exactly that workspace runs, a smaller one is refused."""
    T, K, N, G = 300, 256, 5120, 128
    need = zq.lib().zq_w8a8_linear_workspace(T, K, N, zq.ZQ_OUT_I8_REQUANT)
    assert 4 * (T + 3) <= need < 4 * T * N
    xq, s_tok, Wq, s_grp, bias = _case(T, K, N, G, seed=99)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    q, s = zq.zq_w8a8_linear(dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G, bias=dev(bias), act=zq.ZQ_ACT_GELU,
                             out_kind=zq.ZQ_OUT_I8_REQUANT, workspace=ws)
    q_ref, s_ref = oracle.linear_requant(xq, s_tok, Wq, s_grp, G, bias, oracle.ACT_GELU)
    assert_codes_close(host(q), q_ref)
    assert_scales_close(host(s), s_ref)
    with pytest.raises(zq.ZQError) as e:
        zq.zq_w8a8_linear(dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G, bias=dev(bias), act=zq.ZQ_ACT_GELU,
                          out_kind=zq.ZQ_OUT_I8_REQUANT, workspace=ws[: need - 256])
    assert e.value.status == zq.ZQ_ERR_WORKSPACE
