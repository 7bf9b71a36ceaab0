"""GPU parity of the W8A8 linear (tcgen05 INT8 GEMM + fused dequant
epilogue) against the CPU oracle, through the C ABI.

Shapes cover one tile, several tiles with ragged edges in every dimension
(T not a multiple of 128, N with a half-filled 32-column chunk, K not a
multiple of the 128-byte stage), both operand orders (few tokens swap the
MMA roles) and every output kind."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import (BF16_TOL, F32_TOL, assert_codes_close, assert_dequant_close,
                               assert_scales_close, dequant_magnitude, dev, host)

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


# (T, K, N, G): tokens, reduction, outputs, weight rows per group
GEMM_SHAPES = [
    (128, 128, 256, 16),     # exactly one tile (non-swapped, BN = 256)
    (16, 64, 256, 16),       # the tiny layer: swapped, BN = 16, K < one stage
    (1, 160, 128, 128),      # one token, K = 128 + 32
    (33, 4096, 384, 128),    # swapped, BN = 64 (33 tokens)
    (24, 6144, 1024, 128),   # swapped, BN = 32 (16-column epilogue chunks), split K
    (32, 2048, 272, 16),     # swapped, BN = 32, ragged M tile
    (64, 1040, 272, 16),     # swapped, N % 32 == 16, K tail of 16
    (65, 256, 512, 64),      # first non-swapped T
    (200, 384, 512, 64),     # ragged T
    (300, 208, 400, 80),     # ragged N tile (400 = 256 + 144), K = 208
    (1000, 512, 144, 48),    # BN = 128 path (N < 256)
    (257, 768, 3072, 64),    # BERT W1 shape, ragged T
    (512, 3072, 768, 64),    # BERT W2 shape
]


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


def _ids(shapes):
    return [f"T{t}_K{k}_N{n}_G{g}" for t, k, n, g in shapes]


@pytest.mark.parametrize("T,K,N,G", GEMM_SHAPES, ids=_ids(GEMM_SHAPES))
def test_int32_accumulators_bit_exact(zq, T, K, N, G):
    xq, s_tok, Wq, s_grp, _ = _case(T, K, N, G, seed=T + K + N)
    acc = zq.zq_w8a8_linear(dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G,
                            out_kind=zq.ZQ_OUT_I32_RAW)
    np.testing.assert_array_equal(host(acc), oracle.gemm_i32(xq, Wq))


@pytest.mark.parametrize("T,K,N,G", GEMM_SHAPES, ids=_ids(GEMM_SHAPES))
@pytest.mark.parametrize("act", [0, 1], ids=["none", "gelu"])
def test_dequant_fp32_and_bf16(zq, T, K, N, G, act):
    xq, s_tok, Wq, s_grp, bias = _case(T, K, N, G, seed=3 * T + K + N)
    args = (dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G)
    acc = oracle.gemm_i32(xq, Wq)
    mag = dequant_magnitude(acc, s_tok, s_grp, G, bias)
    y_ref = oracle.dequant(acc, s_tok, s_grp, G, bias, act)
    y32 = zq.zq_w8a8_linear(*args, bias=dev(bias), act=act, out_kind=zq.ZQ_OUT_F32)
    assert_dequant_close(host(y32), y_ref, mag, F32_TOL)
    y16 = zq.zq_w8a8_linear(*args, bias=dev(bias), act=act, out_kind=zq.ZQ_OUT_BF16)
    assert_dequant_close(host(y16), y_ref, mag, BF16_TOL)


@pytest.mark.parametrize("T,K,N,G", GEMM_SHAPES, ids=_ids(GEMM_SHAPES))
def test_dequant_without_bias(zq, T, K, N, G):
    xq, s_tok, Wq, s_grp, _ = _case(T, K, N, G, seed=5 * T + N)
    y = zq.zq_w8a8_linear(dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G, out_kind=zq.ZQ_OUT_F32)
    acc = oracle.gemm_i32(xq, Wq)
    assert_dequant_close(host(y), oracle.dequant(acc, s_tok, s_grp, G, None),
                         dequant_magnitude(acc, s_tok, s_grp, G, None), F32_TOL)


@pytest.mark.parametrize("T,K,N,G", GEMM_SHAPES, ids=_ids(GEMM_SHAPES))
def test_requant_epilogue(zq, T, K, N, G):
    xq, s_tok, Wq, s_grp, bias = _case(T, K, N, G, seed=7 * T + K)
    q2, s2 = zq.zq_w8a8_linear(dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G, bias=dev(bias),
                               act=zq.ZQ_ACT_GELU, out_kind=zq.ZQ_OUT_I8_REQUANT)
    q_ref, s_ref = oracle.linear_requant(xq, s_tok, Wq, s_grp, G, bias, oracle.ACT_GELU)
    assert_codes_close(host(q2), q_ref)
    assert_scales_close(host(s2), s_ref)


def test_group_special_cases(zq):
    """G = 1 (per-row, vector-wise scales) and G = N (one per-tensor scale)."""
    T, K, N = 96, 256, 256
    for G in (1, N):
        xq, s_tok, Wq, s_grp, bias = _case(T, K, N, G, seed=G)
        y = zq.zq_w8a8_linear(dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G, bias=dev(bias),
                              out_kind=zq.ZQ_OUT_F32)
        acc = oracle.gemm_i32(xq, Wq)
        assert_dequant_close(host(y), oracle.dequant(acc, s_tok, s_grp, G, bias),
                             dequant_magnitude(acc, s_tok, s_grp, G, bias), F32_TOL)


def test_extreme_codes_closed_form(zq):
    """All codes +-127: acc = +-127^2 K exactly, also at the largest legal K."""
    for T, K, N in [(128, 2048, 256), (16, 133136, 128)]:
        xq = torch.full((T, K), 127, dtype=torch.int8, device="cuda")
        Wq = torch.full((N, K), 127, dtype=torch.int8, device="cuda")
        Wq[1::2] = -127
        s = torch.ones(T, device="cuda")
        sg = torch.ones(N, device="cuda")
        acc = host(zq.zq_w8a8_linear(xq, s, Wq, sg, 1, out_kind=zq.ZQ_OUT_I32_RAW))
        expect = np.where(np.arange(N) % 2 == 0, 127 * 127 * K, -127 * 127 * K)
        np.testing.assert_array_equal(acc, np.broadcast_to(expect, (T, N)))


def test_overflow_guard_rejects_large_k(zq):
    T, N = 16, 16
    K = zq.ZQ_MAX_K + 8                # next multiple of 16 past the bound
    xq = torch.zeros((T, K), dtype=torch.int8, device="cuda")
    Wq = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    with pytest.raises(zq.ZQError) as e:
        zq.zq_w8a8_linear(xq, torch.ones(T, device="cuda"), Wq, torch.ones(N, device="cuda"), 16,
                          out_kind=zq.ZQ_OUT_I32_RAW)
    assert e.value.status == zq.ZQ_ERR_OVERFLOW


def test_matches_library_int8_matmul_full_coverage(zq):
    """Every accumulator of a 4-wave problem against torch._int_mm (cuBLASLt)."""
    T, K, N = 2048, 1024, 4096
    g = torch.Generator(device="cuda").manual_seed(0)
    xq = torch.randint(-127, 128, (T, K), dtype=torch.int8, device="cuda", generator=g)
    Wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda", generator=g)
    ones_t = torch.ones(T, device="cuda")
    ones_n = torch.ones(N, device="cuda")
    acc = zq.zq_w8a8_linear(xq, ones_t, Wq, ones_n, 1, out_kind=zq.ZQ_OUT_I32_RAW)
    ref = torch._int_mm(xq, Wq.t())
    assert torch.equal(acc, ref)
