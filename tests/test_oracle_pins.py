"""Pins for the CPU oracle: each check ties it to something other than itself.

* hand-worked examples from the pages' rules (``tests/golden/*.txt``);
* closed forms and brute force against library routines (numpy int64
  matmul, torch float64 LayerNorm and GeLU);
* invariants the pages state: codes within [-127, 127], the absmax element
  maps to +-127 ("探秘Transformer系列之（36）— 大模型量化方案" §1.1.2), and the
  rounding error is at most s/2 ("Integer Quantization: Deep Dive",
  quantization error);
* the end-to-end W8A8 linear equals the fake-quantization formulation
  (dequantize each operand, float64 library matmul) and stays within the
  error bound that follows from the s/2 rounding bound against the float
  matmul; plausible mistakes planted in the oracle (on the CPU) break these
  pins.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.golden.fixtures import load_blocks
from w8a8_post_quantized_b200 import inputs


# ---------------------------------------------------------------- quantizer

@pytest.mark.parametrize("block", load_blocks("quantize_vectors.txt"))
def test_quantize_span_hand_examples(block):
    q, s = oracle.quantize_span(block["v"].astype(np.float32))
    np.testing.assert_array_equal(q, block["q"].astype(np.int8))
    assert np.float32(s).tobytes() == np.float32(block["scale"][0]).tobytes()


def _quant_invariants(v, q, s):
    v = v.astype(np.float64)
    amax = np.abs(v).max()
    assert s >= 0
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    if amax == 0:
        assert s == 0 and np.all(q == 0)
        return
    # the absmax element maps to +-127 with its own sign
    i = int(np.argmax(np.abs(v)))
    assert int(q[i]) == (127 if v[i] > 0 else -127)
    # scale is absmax/127 to within one fp32 rounding
    assert abs(float(s) * 127.0 - amax) <= amax * 2.0 ** -23
    # rounding error at most s/2 (plus the fp32 rounding of 127/absmax)
    err = np.abs(v - q.astype(np.float64) * float(s))
    assert np.all(err <= float(s) * 0.5 * (1.0 + 1e-4))


def test_quantize_rows_invariants_random():
    rng = np.random.default_rng(1234)
    Y = rng.standard_t(3.0, size=(64, 384)).astype(np.float32)
    Y[:, [5, 77]] *= 40.0
    Y[7] = 0.0                       # a zero row
    Y[9] = -Y[9]
    q, s = oracle.quantize_rows(Y)
    for t in range(Y.shape[0]):
        _quant_invariants(Y[t], q[t], s[t])


def test_quantize_rows_is_per_token():
    """Scaling one row changes that row's scale only (token-wise, §1.2.2)."""
    rng = np.random.default_rng(5)
    Y = rng.standard_normal((8, 64)).astype(np.float32)
    q0, s0 = oracle.quantize_rows(Y)
    Y2 = Y.copy()
    Y2[3] *= 8.0                      # exact power-of-two scaling
    q1, s1 = oracle.quantize_rows(Y2)
    np.testing.assert_array_equal(np.delete(q1, 3, 0), np.delete(q0, 3, 0))
    np.testing.assert_array_equal(np.delete(s1, 3), np.delete(s0, 3))
    np.testing.assert_array_equal(q1[3], q0[3])
    assert s1[3] == np.float32(8.0) * s0[3]


# ---------------------------------------------------------- weight groups

def _weight_blocks():
    blocks = load_blocks("weight_groups.txt")
    W = blocks[0]["W"]
    return [(W, b) for b in blocks[1:]]


@pytest.mark.parametrize("W,block", _weight_blocks())
def test_weight_groups_hand_examples(W, block):
    G = int(block["G"][0])
    Wq, s = oracle.quantize_weights(W.astype(np.float32), G)
    np.testing.assert_array_equal(Wq, block["Wq"].astype(np.int8))
    np.testing.assert_array_equal(s, block["s_grp"].astype(np.float32))


def test_weight_groups_are_contiguous_output_rows():
    """A large value planted in group g changes group g's scale and codes only."""
    rng = np.random.default_rng(7)
    N, K, G = 96, 48, 16
    W = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    Wq0, s0 = oracle.quantize_weights(W, G)
    W2 = W.copy()
    W2[2 * G + 5, 11] = 3.0          # row 37 lies in group 2
    Wq1, s1 = oracle.quantize_weights(W2, G)
    changed = np.nonzero(s1 != s0)[0]
    np.testing.assert_array_equal(changed, [2])
    rows = np.nonzero(np.any(Wq1 != Wq0, axis=1))[0]
    assert rows.min() >= 2 * G and rows.max() < 3 * G
    assert Wq1[2 * G + 5, 11] == 127
    for g in range(N // G):
        _quant_invariants(W[g * G:(g + 1) * G].ravel(), Wq0[g * G:(g + 1) * G].ravel(), s0[g])


def test_weight_group_special_cases():
    """G = 1 is per-row (vector-wise) quantization; G = N is per-tensor."""
    rng = np.random.default_rng(8)
    W = (0.02 * rng.standard_normal((32, 80))).astype(np.float32)
    Wq1, s1 = oracle.quantize_weights(W, 1)
    amax_rows = np.abs(W).max(axis=1)
    assert np.all(np.abs(s1.astype(np.float64) * 127 - amax_rows) <= amax_rows * 2.0 ** -23)
    WqN, sN = oracle.quantize_weights(W, 32)
    assert sN.shape == (1,)
    assert abs(float(sN[0]) * 127 - np.abs(W).max()) <= np.abs(W).max() * 2.0 ** -23
    _quant_invariants(W.ravel(), WqN.ravel(), sN[0])


# ------------------------------------------------------------------ GEMM

def test_gemm_matches_int64_matmul():
    rng = np.random.default_rng(9)
    for T, K, N in [(1, 16, 1), (7, 48, 13), (33, 160, 70)]:
        xq = rng.integers(-127, 128, size=(T, K), dtype=np.int8)
        Wq = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
        ref = xq.astype(np.int64) @ Wq.astype(np.int64).T
        np.testing.assert_array_equal(oracle.gemm_i32(xq, Wq), ref.astype(np.int32))


def test_gemm_closed_forms():
    K = 64
    ones = np.full((3, K), 127, np.int8)
    np.testing.assert_array_equal(oracle.gemm_i32(ones, ones), np.full((3, 3), 127 * 127 * K))
    np.testing.assert_array_equal(oracle.gemm_i32(ones, -ones), np.full((3, 3), -127 * 127 * K))
    assert 127 * 127 * K == 1032256
    # unit rows pick out one column of Wq: acc[t, o] = Wq[o, t]
    rng = np.random.default_rng(10)
    Wq = rng.integers(-127, 128, size=(5, K), dtype=np.int8)
    eye = np.eye(K, dtype=np.int8)[:8]
    np.testing.assert_array_equal(oracle.gemm_i32(eye, Wq), Wq[:, :8].T.astype(np.int32))


def test_gemm_int32_bound():
    kmax = (2 ** 31 - 1) // (127 * 127)
    assert kmax == 133144
    a = np.full((1, kmax), 127, np.int8)
    assert oracle.gemm_i32(a, a)[0, 0] == 127 * 127 * kmax
    b = np.full((1, kmax + 1), 127, np.int8)
    with pytest.raises(oracle.OracleError):
        oracle.gemm_i32(b, b)


def _dequant_blocks():
    blocks = load_blocks("dequant_linear.txt")
    return [(blocks[0], b) for b in blocks[1:]]


@pytest.mark.parametrize("head,block", _dequant_blocks())
def test_dequant_hand_examples(head, block):
    xq = head["xq"].astype(np.int8)
    Wq = head["Wq"].astype(np.int8)
    acc = oracle.gemm_i32(xq, Wq)
    np.testing.assert_array_equal(acc, head["acc"].astype(np.int32))
    y = oracle.dequant(acc, head["s_tok"].astype(np.float32), block["s_grp"].astype(np.float32),
                       int(block["G"][0]), head["bias"].astype(np.float32))
    np.testing.assert_array_equal(y, block["y"].astype(np.float32))


# --------------------------------------------------------- LayerNorm, GeLU

def _ulps32(a, b):
    a = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(a - b)


def test_layernorm_matches_torch_float64():
    w = inputs.tiny()
    x, g, b = w.x.f32, w.gamma, w.beta
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x).double(), (x.shape[1],),
                                         torch.from_numpy(g).double(),
                                         torch.from_numpy(b).double(), eps=w.eps)
    ref = ref.float().numpy()
    assert _ulps32(oracle.layernorm(x, g, b, w.eps), ref).max() <= 1


def test_layernorm_special_cases():
    H = 32
    g = np.ones(H, np.float32)
    beta = np.linspace(-1, 1, H).astype(np.float32)
    const = np.full((2, H), 3.25, np.float32)
    np.testing.assert_array_equal(oracle.layernorm(const, g, beta, 1e-5), np.stack([beta, beta]))
    # [a, -a, a, -a, ...] with gamma = 1, beta = 0 -> +-a/sqrt(a^2 + eps) -> codes +-127
    a = 2.0
    x = np.tile(np.array([a, -a], np.float32), H // 2)[None, :]
    y = oracle.layernorm(x, g, np.zeros(H, np.float32), 1e-5)
    np.testing.assert_allclose(y[0, :2], [a / np.sqrt(a * a + 1e-5), -a / np.sqrt(a * a + 1e-5)],
                               rtol=1e-7)
    q, s = oracle.ln_quant(x, g, np.zeros(H, np.float32), 1e-5)
    np.testing.assert_array_equal(q[0], np.tile([127, -127], H // 2))


def test_gelu_matches_torch_float64_and_closed_forms():
    v = np.concatenate([np.linspace(-8, 8, 1001), [0.0, 1e-3, -1e-3, 30.0, -30.0]]).astype(np.float32)
    x = v[None, :]
    y = oracle.bias_act(x, None, oracle.ACT_GELU)[0]
    ref = torch.nn.functional.gelu(torch.from_numpy(v).double(), approximate="none").float().numpy()
    assert _ulps32(y, ref).max() <= 1
    assert y[np.where(v == 0)[0][0]] == 0.0
    assert y[np.where(v == 30.0)[0][0]] == np.float32(30.0)
    assert y[np.where(v == -30.0)[0][0]] == 0.0 or abs(y[np.where(v == -30.0)[0][0]]) < 1e-30
    # gelu(x) - gelu(-x) = x
    yn = oracle.bias_act(-x, None, oracle.ACT_GELU)[0]
    np.testing.assert_allclose(y.astype(np.float64) - yn, v, atol=2e-6, rtol=1e-6)


def test_bias_act_identity_is_exact_fp32_sum():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    b = (0.01 * rng.standard_normal(64)).astype(np.float32)
    np.testing.assert_array_equal(oracle.bias_act(x, None, oracle.ACT_NONE), x)
    np.testing.assert_array_equal(oracle.bias_act(x, b, oracle.ACT_NONE), x + b)


def test_dequant_gelu_matches_torch():
    rng = np.random.default_rng(12)
    acc = rng.integers(-200000, 200000, size=(6, 32), dtype=np.int32)
    st = rng.uniform(0.001, 0.05, 6).astype(np.float32)
    sg = rng.uniform(1e-4, 1e-3, 4).astype(np.float32)
    b = (0.01 * rng.standard_normal(32)).astype(np.float32)
    y = oracle.dequant(acc, st, sg, 8, b, oracle.ACT_GELU)
    pre = st.astype(np.float64)[:, None] * np.repeat(sg.astype(np.float64), 8)[None, :] * acc + b
    ref = torch.nn.functional.gelu(torch.from_numpy(pre), approximate="none").float().numpy()
    assert _ulps32(y, ref).max() <= 1


# ----------------------------------------- end-to-end error bound and mutants

def _linear_error_bound(x, W, bias, G, y_q, xq, s_tok, Wq, s_grp):
    """|y_q - (x W^T + b)| <= sum_k |x_k| s_w/2 + |w_hat_k| s_x/2, from the
    per-element rounding bound s/2 on both operands."""
    x64 = x.astype(np.float64)
    y_fp = x64 @ W.astype(np.float64).T + bias
    sw = np.repeat(s_grp.astype(np.float64), G)                 # per output row
    w_hat = Wq.astype(np.float64) * sw[:, None]
    bound = (np.abs(x64).sum(1)[:, None] * sw[None, :] * 0.5
             + s_tok.astype(np.float64)[:, None] * 0.5 * np.abs(w_hat).sum(1)[None, :])
    slack = 1e-5 * (np.abs(x64) @ np.abs(W.astype(np.float64)).T) + 1e-6
    return np.abs(y_q.astype(np.float64) - y_fp), bound * (1 + 1e-3) + slack


def _tiny_linear():
    w = inputs.tiny()
    lin = w.layers[0]
    x = w.x.f32
    xq, s_tok = oracle.quantize_rows(x)
    Wq, s_grp = oracle.quantize_weights(lin.W, lin.group_rows)
    return w, lin, x, xq, s_tok, Wq, s_grp


def test_linear_within_rounding_error_bound():
    w, lin, x, xq, s_tok, Wq, s_grp = _tiny_linear()
    y = oracle.linear(xq, s_tok, Wq, s_grp, lin.group_rows, lin.bias)
    err, bound = _linear_error_bound(x, lin.W, lin.bias, lin.group_rows, y, xq, s_tok, Wq, s_grp)
    assert np.all(err <= bound)


def _fake_quant_gap(y_q, xq, s_tok, Wq, s_grp, G, bias):
    """Fake quantization ("Integer Quantization: Deep Dive", 量化模拟): dequantize
    each operand (x = s * x_int), then multiply in float64 with a library
    matmul.  Dequantizing after the integer GEMM must give the same numbers
    up to fp32 output rounding."""
    x_hat = xq.astype(np.float64) * s_tok.astype(np.float64)[:, None]
    w_hat = Wq.astype(np.float64) * np.repeat(s_grp.astype(np.float64), G)[:, None]
    ref = x_hat @ w_hat.T + bias.astype(np.float64)
    scale = np.abs(x_hat) @ np.abs(w_hat).T + np.abs(bias.astype(np.float64))
    return np.abs(y_q.astype(np.float64) - ref) / (scale + 1e-30)


def test_linear_matches_fake_quantization():
    w, lin, x, xq, s_tok, Wq, s_grp = _tiny_linear()
    y = oracle.linear(xq, s_tok, Wq, s_grp, lin.group_rows, lin.bias)
    assert _fake_quant_gap(y, xq, s_tok, Wq, s_grp, lin.group_rows, lin.bias).max() <= 2 ** -22


MUTANTS = ["group_index_mod", "transposed_scales", "dropped_bias", "sign_flip_row",
           "wrong_token_scale"]


@pytest.mark.parametrize("mutant", MUTANTS)
def test_pins_catch_planted_mistakes(mutant):
    """Plausible oracle mistakes, planted on the CPU, must break the pins:
    every mutant breaks the fake-quantization identity, and every mistake in
    the scales also breaks the s/2 error bound against the float matmul."""
    w, lin, x, xq, s_tok, Wq, s_grp = _tiny_linear()
    G = lin.group_rows
    acc = oracle.gemm_i32(xq, Wq)
    bias = lin.bias
    if mutant == "group_index_mod":           # g(o) = o mod n_groups instead of o // G
        n = len(s_grp)
        sg_bad = s_grp[np.arange(lin.W.shape[0]) % n]
        y = oracle.dequant(acc, s_tok, sg_bad, 1, bias)
    elif mutant == "transposed_scales":       # groups read in reverse order
        y = oracle.dequant(acc, s_tok, s_grp[::-1].copy(), G, bias)
    elif mutant == "dropped_bias":
        y = oracle.dequant(acc, s_tok, s_grp, G, None)
    elif mutant == "sign_flip_row":           # a sign error on one weight row
        Wq2 = Wq.copy()
        Wq2[3] = -Wq2[3]
        y = oracle.linear(xq, s_tok, Wq2, s_grp, G, bias)
    else:                                     # token scales shifted by one row
        y = oracle.dequant(acc, np.roll(s_tok, 1), s_grp, G, bias)
    assert _fake_quant_gap(y, xq, s_tok, Wq, s_grp, G, bias).max() > 1e-3
    if mutant in ("group_index_mod", "transposed_scales", "wrong_token_scale", "sign_flip_row"):
        err, bound = _linear_error_bound(x, lin.W, bias, G, y, xq, s_tok, Wq, s_grp)
        assert np.any(err > bound)


def test_ln_quant_and_requant_compose_pinned_steps():
    """The fused compositions equal the pinned steps run one after another."""
    w = inputs.tiny()
    x = w.x.f32
    ln_ref = torch.nn.functional.layer_norm(torch.from_numpy(x).double(), (x.shape[1],),
                                            torch.from_numpy(w.gamma).double(),
                                            torch.from_numpy(w.beta).double(), eps=w.eps)
    q_ref, s_ref = oracle.quantize_rows(ln_ref.float().numpy())
    q, s = oracle.ln_quant(x, w.gamma, w.beta, w.eps)
    np.testing.assert_array_equal(q, q_ref)
    np.testing.assert_array_equal(s, s_ref)
    lin = w.layers[0]
    Wq, sg = oracle.quantize_weights(lin.W, lin.group_rows)
    q2, s2 = oracle.linear_requant(q, s, Wq, sg, lin.group_rows, lin.bias, oracle.ACT_GELU)
    acc = q.astype(np.int64) @ Wq.astype(np.int64).T
    pre = (s.astype(np.float64)[:, None] * np.repeat(sg.astype(np.float64), lin.group_rows)[None]
           * acc + lin.bias)
    h = torch.nn.functional.gelu(torch.from_numpy(pre), approximate="none").float().numpy()
    q2_ref, s2_ref = oracle.quantize_rows(h)
    np.testing.assert_array_equal(q2, q2_ref)
    np.testing.assert_array_equal(s2, s2_ref)
