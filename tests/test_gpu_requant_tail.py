"""The requantizing linear (cluster-fused dequant + bias + GeLU + per-token
requant) when the 128-row blocks do not divide evenly over the co-resident
clusters, so the clusters run a partial last round (and, for ragged T, a
partial last block).  Parity with the CPU oracle on every row of the last two
blocks and a sample of the others ("探秘Transformer系列之（36）— 大模型量化方案"
§1.2.2: one dynamic scale per token over the whole output row)."""
import numpy as np
import pytest

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


# 128-row blocks over 22 co-resident clusters of 6: T = 4096 -> 32 blocks
# (a second round of 10); 2900 -> 23 (one block in round two, ragged);
# 4000 -> 32 with a ragged last block; 5504 -> 43; 6000 -> 47 (a third round)
@pytest.mark.parametrize("T", [4096, 2900, 4000, 5504, 6000])
def test_requant_tail_rows(zq, T):
    K, N, G = 768, 3072, 64
    rng = np.random.default_rng(T)
    x = rng.standard_normal((T, K)).astype(np.float32)
    x[:, rng.permutation(K)[:6]] *= 20.0
    W = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    xq_ref, st_ref = oracle.quantize_rows(x)
    Wq_ref, sg_ref = oracle.quantize_weights(W, G)
    q, st = zq.zq_w8a8_linear(dev(xq_ref), dev(st_ref), dev(Wq_ref), dev(sg_ref), G, bias=dev(bias),
                              act=zq.ZQ_ACT_GELU, out_kind=zq.ZQ_OUT_I8_REQUANT)
    qh, sth = host(q), host(st)
    # every row of the last two 128-row blocks, plus a seeded sample
    tail = np.arange(max(0, (T - 1) // 128 * 128 - 128), T)
    rows = np.unique(np.concatenate([tail, sample_rows(T, 48, seed=T)]))
    q_ref, s_ref = oracle.linear_requant(xq_ref[rows], st_ref[rows], Wq_ref, sg_ref, G, bias, oracle.ACT_GELU)
    assert_codes_close(qh[rows], q_ref)
    assert_scales_close(sth[rows], s_ref)
    # invariants on all rows: each row's absmax code is +-127
    assert np.all(np.abs(qh).max(axis=1) == 127)
