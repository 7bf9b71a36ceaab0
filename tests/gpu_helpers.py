"""Shared helpers for the GPU parity tests: moving seeded inputs to the
device and the comparison rules.

Tolerances (the comparison contract):
  * quantizer codes/scales from identical fp32 input: bit-exact;
  * codes after fp32 LayerNorm / GeLU on the GPU versus the fp64 oracle:
    at most 0.1% of codes differ, each by +-1; scales within 1e-5 relative;
  * int32 accumulators: bit-exact;
  * dequantized outputs given the same accumulators: |y - ref| <= tol *
    (|s_tok * s_grp * acc| + |bias|), tol = 1e-5 for fp32, 1e-2 for bf16
    (the term magnitude keeps the bound meaningful under cancellation).
"""
import numpy as np
import torch

from w8a8_post_quantized_b200.inputs import Activation

CODE_MISMATCH_FRAC = 1e-3
SCALE_RTOL = 1e-5
F32_TOL = 1e-5
BF16_TOL = 1e-2


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def dev_act(a: Activation) -> torch.Tensor:
    if a.bf16 is not None:
        return torch.from_numpy(a.bf16.view(np.int16)).cuda().view(torch.bfloat16)
    return dev(a.f32)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def assert_codes_close(q_gpu, q_ref, max_frac=CODE_MISMATCH_FRAC):
    d = q_gpu.astype(np.int32) - q_ref.astype(np.int32)
    assert np.abs(d).max(initial=0) <= 1, f"code differs by {np.abs(d).max()}"
    frac = np.count_nonzero(d) / max(d.size, 1)
    assert frac <= max_frac, f"{frac:.3%} of codes differ (limit {max_frac:.3%})"
    return frac


def assert_scales_close(s_gpu, s_ref, rtol=SCALE_RTOL):
    s_gpu = s_gpu.astype(np.float64)
    s_ref = s_ref.astype(np.float64)
    np.testing.assert_array_less(np.abs(s_gpu - s_ref), rtol * np.abs(s_ref) + 1e-38)


def dequant_magnitude(acc, s_tok, s_grp, G, bias):
    """|s_tok[t] * s_grp[o // G] * acc[t, o]| + |bias[o]| (float64)."""
    mag = (np.abs(s_tok.astype(np.float64))[:, None]
           * np.repeat(np.abs(s_grp.astype(np.float64)), G)[None, :]
           * np.abs(acc.astype(np.float64)))
    if bias is not None:
        mag = mag + np.abs(bias.astype(np.float64))[None, :]
    return mag


def assert_dequant_close(y_gpu, y_ref, mag, tol):
    err = np.abs(y_gpu.astype(np.float64) - y_ref.astype(np.float64))
    bad = err > tol * mag + 1e-30
    assert not bad.any(), (f"{bad.sum()} outputs outside tolerance; worst ratio "
                           f"{(err / (mag + 1e-30)).max():.3e}")


def sample_rows(T, n=48, seed=0):
    """First, last and a seeded spread of rows in between (sorted, unique)."""
    rng = np.random.default_rng(seed)
    rows = {0, T - 1, T // 2}
    rows.update(rng.choice(T, size=min(n, T), replace=False).tolist())
    return np.array(sorted(rows))
