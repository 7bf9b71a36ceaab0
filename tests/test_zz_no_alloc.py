"""The requantizing linear that needs no caller scratch and allocates nothing
(zq_w8a8_linear_requant_noalloc), for callers that cannot obtain device
memory themselves -- e.g. plugins of a host framework that owns every device
allocation, or serving loops where cudaMalloc is not allowed after start-up.

It takes the same kernels as the workspace-taking entry point
zq_w8a8_linear(..., ZQ_OUT_I8_REQUANT), with the library's fixed scratch
array in place of the workspace: per-token absmax words and row-block
counters for rows wider than 4096 features, the fp32 output for at most 64
tokens, nothing at all for the cluster kernel.  The GPU test calls it
through the C ABI on several problems in a row, each route twice (the array
keeps the previous call's contents when the next starts), and compares each
result with the CPU oracle's requantizing linear and with the
workspace-taking entry point, within the tolerances the other tests use.
This file is collected last so that a run stopping at the first failure
has already run every other test; it also passes on its own in a
fresh process (the first call does the per-device set-up)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import assert_codes_close, assert_scales_close, dev, host, sample_rows
from w8a8_post_quantized_b200 import zq


def _case(T, K, N, G, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(4.0, size=(T, K)).astype(np.float32)
    x[:, rng.permutation(K)[: max(1, K // 100)]] *= 25.0
    W = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    xq, s_tok = oracle.quantize_rows(x)
    Wq, s_grp = oracle.quantize_weights(W, G)
    return xq, s_tok, Wq, s_grp, bias


def _call_noalloc(xq, s_tok, Wq, s_grp, G, bias, y, s_out):
    """Direct C-ABI call with caller-provided outputs (nothing allocated here)."""
    T, K = xq.shape
    N = Wq.shape[0]
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return zq.lib().zq_w8a8_linear_requant_noalloc(P(xq), P(s_tok), T, K, P(Wq), P(s_grp), N, G,
                                                   P(bias), zq.ZQ_ACT_GELU, P(y), P(s_out), stream)


@pytest.mark.gpu
def test_noalloc_requant_matches_oracle_and_workspace_entry_point():
    # (T, K, N, G, seed, rows checked against the oracle: None = all)
    cases = [(300, 256, 5120, 128, 13, None),  # rows wider than 4096: absmax words + counters
             (48, 512, 2048, 64, 15, None),    # 48 tokens: the fp32 output in the array
             (4096, 768, 3072, 64, 11, 96),    # the BERT W1 layer: the cluster kernel, no scratch
             (300, 256, 5120, 128, 14, None),  # wide rows again, over the fp32 route's contents
             (48, 512, 2048, 64, 16, None),    # 48 tokens again, new data
             (2048, 1024, 16384, 128, 17, 32)] # GPT-J FFN-up width, 2048 tokens
    for T, K, N, G, seed, n_rows in cases:
        xq, s_tok, Wq, s_grp, bias = _case(T, K, N, G, seed)
        d = [dev(a) for a in (xq, s_tok, Wq, s_grp, bias)]
        y = torch.empty((T, N), dtype=torch.int8, device="cuda")
        s_out = torch.empty(T, dtype=torch.float32, device="cuda")
        assert _call_noalloc(d[0], d[1], d[2], d[3], G, d[4], y, s_out) == zq.ZQ_OK
        zq.zq_device_status()
        qh, sh = host(y), host(s_out)
        # against the oracle (all rows, or the last block and a seeded sample)
        rows = (np.arange(T) if n_rows is None else
                np.unique(np.concatenate([np.arange(T - 128, T), sample_rows(T, n_rows, seed=seed)])))
        q_ref, s_ref = oracle.linear_requant(xq[rows], s_tok[rows], Wq, s_grp, G, bias, oracle.ACT_GELU)
        assert_codes_close(qh[rows], q_ref)
        assert_scales_close(sh[rows], s_ref)
        # against the workspace-taking entry point (every row)
        ref_y, ref_s = zq.zq_w8a8_linear(d[0], d[1], d[2], d[3], G, bias=d[4], act=zq.ZQ_ACT_GELU,
                                         out_kind=zq.ZQ_OUT_I8_REQUANT)
        zq.zq_device_status()
        assert_codes_close(qh, host(ref_y))
        assert_scales_close(sh, host(ref_s))


def test_noalloc_rejects_problems_beyond_its_scratch():
    """Host-side check, before anything is enqueued (fake pointers are never used)."""
    A = 0x7F0000000000
    T, N = 64, 300000                        # 64 tokens: 76.8 MB of fp32 output, does not fit
    rc = zq.lib().zq_w8a8_linear_requant_noalloc(A, A, T, 768, A, A, N, 16, None, 1, A, A, None)
    assert rc == zq.ZQ_ERR_SCRATCH
    T, N = 20 << 20, 8192                    # wide rows: 80 MiB of absmax words alone
    rc = zq.lib().zq_w8a8_linear_requant_noalloc(A, A, T, 64, A, A, N, 64, None, 1, A, A, None)
    assert rc == zq.ZQ_ERR_SCRATCH
    assert zq.ZQ_NOALLOC_SCRATCH_BYTES == 64 << 20
    assert zq.lib().zq_w8a8_linear_requant_noalloc(None, A, 4, 64, A, A, 16, 16, None, 1, A, A,
                                                   None) == zq.ZQ_ERR_NULL
