"""GPU parity of the few-token linear (T <= 64, weights on the MMA's M side,
tokens as its N side) on its even-split route, against the CPU oracle,
through the C ABI.  The (weight tile, k-block) iterations are cut into equal
contiguous ranges, one per SM; a tile cut by a range boundary is summed from
int32 partials that other CTAs publish in the workspace.

ZQ_EVEN_SPLIT=on forces that route for every T <= 64 (the default takes it
when there are at least as many weight tiles as SMs); ZQ_EVEN_SPLIT=off
forces the split-K clusters.  Both must give the oracle's int32 accumulators
exactly and the same dequantized values.

Shapes cut tiles everywhere they can be cut: one tile spread over a hundred
CTAs (one k-block each), tiles spread over a few CTAs with a boundary inside
a tile, ranges holding whole tiles plus a cut one, ragged N and K edges, and
the decode layer at full size on sampled columns."""
import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import (BF16_TOL, F32_TOL, assert_dequant_close, dequant_magnitude, dev,
                               host)

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


# (T, K, N, G)
FEW_TOKEN_SHAPES = [
    (16, 16384, 128, 128),   # one tile, 128 k-blocks: one per CTA, 127 partials summed
    (1, 128, 16, 16),        # one iteration in all: a grid of one CTA
    (33, 2048, 1040, 16),    # 9 tiles x 16 k-blocks, ragged last tile (N % 128 = 16)
    (64, 1040, 2048, 64),    # K tail of 16 bytes in the last k-block
    (8, 3072, 4096, 128),    # 32 tiles x 24 k-blocks: 6 iterations a CTA, boundaries mid-tile
    (24, 768, 16384, 128),   # 128 tiles x 6 k-blocks: whole tiles plus cut ones in a range
    (48, 4096, 2304, 256),   # 18 tiles x 32 k-blocks, 4 or 5 CTAs a tile
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


ALL_SHAPES = FEW_TOKEN_SHAPES


def test_workspace_is_offered_where_the_split_is_taken(zq, monkeypatch):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    monkeypatch.delenv("ZQ_EVEN_SPLIT", raising=False)
    # decode layer: 192 weight tiles, every range holds a whole tile
    ws = zq.zq_w8a8_linear_workspace(16, 6144, 24576, zq.ZQ_OUT_BF16)
    assert sms * 128 * 64 * 4 <= ws < 8 << 20
    # 8192 x 8192 with 16 tokens: 64 weight tiles, fewer than SMs: split-K clusters
    assert zq.zq_w8a8_linear_workspace(16, 8192, 8192, zq.ZQ_OUT_BF16) == 0
    # more tokens: whole tiles, no workspace
    assert zq.zq_w8a8_linear_workspace(65, 6144, 24576, zq.ZQ_OUT_BF16) == 0
    monkeypatch.setenv("ZQ_EVEN_SPLIT", "off")
    assert zq.zq_w8a8_linear_workspace(16, 6144, 24576, zq.ZQ_OUT_BF16) == 0
    monkeypatch.setenv("ZQ_EVEN_SPLIT", "on")
    assert zq.zq_w8a8_linear_workspace(16, 8192, 8192, zq.ZQ_OUT_BF16) > 0
    assert zq.zq_w8a8_linear_workspace(65, 6144, 24576, zq.ZQ_OUT_BF16) == 0


@pytest.mark.parametrize("T,K,N,G", ALL_SHAPES, ids=_ids(ALL_SHAPES))
def test_accumulators_bit_exact_on_both_routes(zq, monkeypatch, T, K, N, G):
    xq, s_tok, Wq, s_grp, _ = _case(T, K, N, G, seed=11 * T + K + N)
    args = (dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G)
    ref = oracle.gemm_i32(xq, Wq)
    for mode in ("on", "off"):
        monkeypatch.setenv("ZQ_EVEN_SPLIT", mode)
        acc = zq.zq_w8a8_linear(*args, out_kind=zq.ZQ_OUT_I32_RAW)
        np.testing.assert_array_equal(host(acc), ref, err_msg=f"ZQ_EVEN_SPLIT={mode}")


@pytest.mark.parametrize("T,K,N,G", ALL_SHAPES, ids=_ids(ALL_SHAPES))
@pytest.mark.parametrize("act", [0, 1], ids=["none", "gelu"])
def test_dequant_on_both_routes(zq, monkeypatch, T, K, N, G, act):
    xq, s_tok, Wq, s_grp, bias = _case(T, K, N, G, seed=13 * T + K + N)
    args = (dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G)
    acc = oracle.gemm_i32(xq, Wq)
    mag = dequant_magnitude(acc, s_tok, s_grp, G, bias)
    y_ref = oracle.dequant(acc, s_tok, s_grp, G, bias, act)
    monkeypatch.setenv("ZQ_EVEN_SPLIT", "on")
    y32 = zq.zq_w8a8_linear(*args, bias=dev(bias), act=act, out_kind=zq.ZQ_OUT_F32)
    assert_dequant_close(host(y32), y_ref, mag, F32_TOL)
    y16 = zq.zq_w8a8_linear(*args, bias=dev(bias), act=act, out_kind=zq.ZQ_OUT_BF16)
    assert_dequant_close(host(y16), y_ref, mag, BF16_TOL)
    # split-K clusters: same accumulators, same epilogue arithmetic, same fp32 values
    monkeypatch.setenv("ZQ_EVEN_SPLIT", "off")
    y32b = zq.zq_w8a8_linear(*args, bias=dev(bias), act=act, out_kind=zq.ZQ_OUT_F32)
    np.testing.assert_array_equal(host(y32b), host(y32))


def test_no_workspace_takes_the_other_route(zq, monkeypatch):
    """The workspace is optional for these output kinds: without one the
    call splits K over clusters, same results."""
    monkeypatch.setenv("ZQ_EVEN_SPLIT", "on")
    for T, K, N, G in [(16, 4096, 2048, 128), (64, 2048, 1024, 128)]:
        xq, s_tok, Wq, s_grp, _ = _case(T, K, N, G, seed=T)
        args = (dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G)
        ref = oracle.gemm_i32(xq, Wq)
        none = torch.empty(0, dtype=torch.uint8, device="cuda")
        small = torch.empty(zq.zq_w8a8_linear_workspace(T, K, N, zq.ZQ_OUT_I32_RAW) - 256,
                            dtype=torch.uint8, device="cuda")
        for ws in (none, small):
            acc = zq.zq_w8a8_linear(*args, out_kind=zq.ZQ_OUT_I32_RAW, workspace=ws)
            np.testing.assert_array_equal(host(acc), ref)


@pytest.mark.parametrize("T,K,N", [(16, 4096, 2048), (40, 2048, 1024)])
def test_repeated_calls_reuse_the_workspace(zq, monkeypatch, T, K, N):
    """The ready counters are cleared before every call: back-to-back calls on
    one workspace (no host synchronisation between them) stay exact."""
    monkeypatch.setenv("ZQ_EVEN_SPLIT", "on")
    G = 128
    xq, s_tok, Wq, s_grp, _ = _case(T, K, N, G, seed=99)
    args = (dev(xq), dev(s_tok), dev(Wq), dev(s_grp), G)
    ws = torch.empty(zq.zq_w8a8_linear_workspace(T, K, N, zq.ZQ_OUT_I32_RAW), dtype=torch.uint8,
                     device="cuda")
    outs = [zq.zq_w8a8_linear(*args, out_kind=zq.ZQ_OUT_I32_RAW, workspace=ws) for _ in range(8)]
    ref = oracle.gemm_i32(xq, Wq)
    for o in outs:
        np.testing.assert_array_equal(host(o), ref)


def test_neox_decode_layer_sampled(zq, monkeypatch):
    """The decode layer at full size (16 tokens, 6144 -> 24576, G = 256,
    GeLU), on the default route (the even split: 192 weight tiles): bf16
    outputs of 512 sampled columns against the oracle on their weight rows;
    the whole int32 product against the split-K clusters."""
    monkeypatch.delenv("ZQ_EVEN_SPLIT", raising=False)
    T, K, N, G = 16, 6144, 24576, 256
    rng = np.random.default_rng(2024)
    x = rng.standard_t(4.0, size=(T, K)).astype(np.float32)
    xq, s_tok = oracle.quantize_rows(x)
    g = torch.Generator(device="cuda").manual_seed(5)
    Wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda", generator=g)
    s_grp = (torch.rand(N // G, device="cuda", generator=g) + 0.5) * 1e-3
    bias = 0.01 * torch.randn(N, device="cuda", generator=g)
    args = (dev(xq), dev(s_tok), Wq, s_grp, G)
    y = zq.zq_w8a8_linear(*args, bias=bias, act=1, out_kind=zq.ZQ_OUT_BF16)
    cols = np.sort(rng.choice(N, 512, replace=False))
    acc = oracle.gemm_i32(xq, host(Wq)[cols])
    sg = host(s_grp)[cols // G]
    b = host(bias)[cols]
    # the sampled columns as a layer of their own with one row per group
    y_ref = oracle.dequant(acc, s_tok, sg, 1, b, oracle.ACT_GELU)
    assert_dequant_close(host(y)[:, cols], y_ref, dequant_magnitude(acc, s_tok, sg, 1, b), BF16_TOL)
    a_model = zq.zq_w8a8_linear(*args, out_kind=zq.ZQ_OUT_I32_RAW)
    monkeypatch.setenv("ZQ_EVEN_SPLIT", "off")
    a_split = zq.zq_w8a8_linear(*args, out_kind=zq.ZQ_OUT_I32_RAW)
    assert torch.equal(a_model, a_split)
    np.testing.assert_array_equal(host(a_model)[:, cols], acc)


def test_largest_k_closed_form(zq, monkeypatch):
    """All codes +-127 at the largest legal K (a multiple of 16, its last
    k-block 16 bytes) through the even split: one weight tile's 1041 k-blocks
    spread over the SMs (about 8 a CTA, so about 130 partial sums per
    output), acc = +-127^2 K exactly, and the same with a ragged second tile
    (N = 144)."""
    monkeypatch.setenv("ZQ_EVEN_SPLIT", "on")
    K = zq.ZQ_MAX_K // 16 * 16
    for T, N in [(16, 128), (64, 144)]:
        xq = torch.full((T, K), 127, dtype=torch.int8, device="cuda")
        Wq = torch.full((N, K), 127, dtype=torch.int8, device="cuda")
        Wq[1::2] = -127
        acc = host(zq.zq_w8a8_linear(xq, torch.ones(T, device="cuda"), Wq, torch.ones(N, device="cuda"), 16,
                                     out_kind=zq.ZQ_OUT_I32_RAW))
        expect = np.where(np.arange(N) % 2 == 0, 127 * 127 * K, -127 * 127 * K)
        np.testing.assert_array_equal(acc, np.broadcast_to(expect, (T, N)))
