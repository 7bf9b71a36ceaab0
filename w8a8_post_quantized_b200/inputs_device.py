"""Seeded synthetic workloads drawn on the GPU, for the benchmark only.

The same shapes and value distributions as ``inputs.py`` (which draws them
with numpy on the host and feeds both the CUDA path and the CPU oracle), but
drawn with torch's counter-based CUDA generator, so the large benchmark
inputs (up to 65536 x 12288 activations, 24576 x 6144 weights) take
milliseconds instead of minutes to make.  The bytes differ from the numpy
recipe's; the distributions do not.  Parity tests never use this module.

Like ``inputs.py`` this module holds only random-number recipes and data
encoding, none of the method's arithmetic.  Student-t(nu) for integer nu is
drawn as Z / sqrt(V / nu) with V the sum of nu squared standard normals (a
chi-squared variable with nu degrees of freedom).  bf16 values are the fp32
draws rounded to nearest even (torch's conversion).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

EPS = 1e-5
ROW_CHUNK = 2048          # rows drawn at a time, so fp32 temporaries stay small


@dataclass
class DevLinear:
    W: torch.Tensor       # fp32 [N, K]
    bias: torch.Tensor    # fp32 [N]
    group_rows: int


@dataclass
class DevWorkload:
    name: str
    x: torch.Tensor       # bf16 or fp32 [T, K]
    gamma: torch.Tensor | None
    beta: torch.Tensor | None
    layers: list = field(default_factory=list)
    act: int = 0
    out: str = "bf16"
    eps: float = EPS


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(g, shape, device, std=1.0):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).mul_(std)


def _student_t(g, shape, nu, device):
    z = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    v = torch.zeros(shape, device=device, dtype=torch.float32)
    for _ in range(nu):
        e = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        v.addcmul_(e, e)
    return z.div_(v.div_(nu).sqrt_())


def _activation(g, T, H, device, kind, scale=1.0, outliers=0, factor=1.0):
    """bf16 [T, H]; rows drawn in chunks; `outliers` channels (a seeded
    permutation, the same for every token) multiplied by `factor`."""
    x = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    ch = None
    if outliers:
        ch = torch.randperm(H, generator=g, device=device)[:outliers].sort().values
    for r0 in range(0, T, ROW_CHUNK):
        rows = min(ROW_CHUNK, T - r0)
        if kind == "normal":
            v = _normal(g, (rows, H), device)
        else:
            v = _student_t(g, (rows, H), kind, device)
        if scale != 1.0:
            v.mul_(scale)
        if ch is not None:
            v[:, ch] *= factor
        x[r0:r0 + rows] = v.to(torch.bfloat16)
    return x


def _ln_params(g, H, device):
    return 1.0 + _normal(g, (H,), device, 0.1), _normal(g, (H,), device, 0.1)


def gptj_qkv(device, seed=2, T=2048):
    g = _gen(seed, device)
    H, N = 4096, 12288
    x = _activation(g, T, H, device, 4, scale=0.5, outliers=8, factor=50.0)
    gamma, beta = _ln_params(g, H, device)
    lo, hi = math.log(0.1), math.log(10.0)
    m = torch.rand(N, 1, generator=g, device=device).mul_(hi - lo).add_(lo).exp_()
    W = _normal(g, (N, H), device, 0.015).mul_(m)
    bias = _normal(g, (N,), device, 0.01)
    return DevWorkload(f"gptj_6b_qkv_{T}x4096x12288_g128", x, gamma, beta, [DevLinear(W, bias, 128)], act=0)


def gptj_ffn(device, seed=4, T=2048):
    """The GPT-J-6B MLP: LN -> 4096 -> 16384 (GeLU, requantized per token) ->
    4096.  Its first linear is wider than 4096 outputs."""
    g = _gen(seed, device)
    H, F = 4096, 16384
    x = _activation(g, T, H, device, 4, scale=0.5, outliers=8, factor=50.0)
    gamma, beta = _ln_params(g, H, device)
    W1 = _normal(g, (F, H), device, 0.015)
    b1 = _normal(g, (F,), device, 0.01)
    W2 = _normal(g, (H, F), device, 0.015)
    b2 = _normal(g, (H,), device, 0.01)
    return DevWorkload(f"gptj_6b_ffn_block_{T}x4096x16384_g128", x, gamma, beta,
                       [DevLinear(W1, b1, 128), DevLinear(W2, b2, 128)], act=1)


def neox_decode(device, seed=3, T=16):
    g = _gen(seed, device)
    H, N = 6144, 24576
    x = _activation(g, T, H, device, "normal", outliers=31, factor=40.0)
    W = _normal(g, (N, H), device, 0.01)
    bias = _normal(g, (N,), device, 0.01)
    return DevWorkload(f"neox_20b_ffn_up_decode_{T}x6144x24576_g256", x, None, None,
                       [DevLinear(W, bias, 256)], act=1)


def gemm_sweep_point(device, M, index, K=8192, N=8192):
    g = _gen(100 + index, device)
    x = _activation(g, M, K, device, 3)
    W = _normal(g, (N, K), device, 0.02)
    bias = _normal(g, (N,), device, 0.01)
    return DevWorkload(f"gemm_sweep_{M}x{K}x{N}_g128", x, None, None, [DevLinear(W, bias, 128)], act=0)


def ln_sweep_point(device, T, H, index):
    g = _gen(100 + index, device)
    x = _activation(g, T, H, device, 3)
    gamma, beta = _ln_params(g, H, device)
    return DevWorkload(f"ln_quant_sweep_{T}x{H}", x, gamma, beta)
