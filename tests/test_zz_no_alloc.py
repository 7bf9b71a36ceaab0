"""The requantizing linear that needs no caller scratch and allocates nothing
(zq_w8a8_linear_requant_noalloc), for callers that cannot obtain device
memory themselves -- e.g. plugins of a host framework that owns every device
allocation, or serving loops where cudaMalloc is not allowed after start-up.

The GPU test calls it through the C ABI twice in a row (the library's fixed
scratch array keeps the first call's contents when the second starts) and
compares each result with the workspace-taking entry point,
zq_w8a8_linear(..., ZQ_OUT_I8_REQUANT), within the tolerances the other
tests use.  This file is collected last so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process (the first call does the per-device set-up)."""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_helpers import assert_codes_close, assert_scales_close, host
from w8a8_post_quantized_b200 import zq


def _inputs(T, K, N, G, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    xq = torch.randint(-127, 128, (T, K), dtype=torch.int8, device="cuda", generator=g)
    Wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda", generator=g)
    s_tok = torch.rand(T, device="cuda", generator=g) * 0.05 + 1e-3
    s_grp = torch.rand(N // G, device="cuda", generator=g) * 1e-3 + 1e-5
    bias = torch.randn(N, device="cuda", generator=g) * 0.01
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
def test_noalloc_requant_matches_workspace_entry_point_twice():
    cases = [(4096, 768, 3072, 64, 11),     # the BERT W1 layer: 48 MiB of the 64 MiB array
             (300, 512, 400, 80, 12)]       # smaller, ragged, run second over stale contents
    outs = []
    for T, K, N, G, seed in cases:
        xq, s_tok, Wq, s_grp, bias = _inputs(T, K, N, G, seed)
        y = torch.empty((T, N), dtype=torch.int8, device="cuda")
        s_out = torch.empty(T, dtype=torch.float32, device="cuda")
        assert _call_noalloc(xq, s_tok, Wq, s_grp, G, bias, y, s_out) == zq.ZQ_OK
        zq.zq_device_status()
        ref_y, ref_s = zq.zq_w8a8_linear(xq, s_tok, Wq, s_grp, G, bias=bias, act=zq.ZQ_ACT_GELU,
                                         out_kind=zq.ZQ_OUT_I8_REQUANT)
        zq.zq_device_status()
        assert_codes_close(host(y), host(ref_y))
        assert_scales_close(host(s_out), host(ref_s))
        outs.append(host(s_out))
    assert outs[0].shape != outs[1].shape


def test_noalloc_rejects_problems_beyond_its_scratch():
    """Host-side check, before anything is enqueued (fake pointers are never used)."""
    A = 0x7F0000000000
    T, N = 4096, 4096                        # 64 MiB of fp32 output alone: does not fit
    rc = zq.lib().zq_w8a8_linear_requant_noalloc(A, A, T, 768, A, A, N, 64, None, 1, A, A, None)
    assert rc == zq.ZQ_ERR_SCRATCH
    assert zq.ZQ_NOALLOC_SCRATCH_BYTES == 64 << 20
    assert zq.lib().zq_w8a8_linear_requant_noalloc(None, A, 4, 64, A, A, 16, 16, None, 1, A, A,
                                                   None) == zq.ZQ_ERR_NULL
