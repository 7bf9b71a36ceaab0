"""Seeded synthetic workloads for the W8A8 linear path.

This module holds only random-number recipes and data encoding (fp32 ->
bf16 bit patterns, round-to-nearest-even).  It contains none of the
method's arithmetic, so both the CUDA path and the CPU oracle can take their
inputs from it.  numpy only; no torch, no CUDA.

Every generator draws from ``numpy.random.default_rng(seed)`` in a fixed
order, so the same seed always gives the same bytes.

Workloads (layer shapes of public model families; no weights are loaded):
  tiny        x fp32 [16, 64] ~N(0,1), channels 3 and 41 scaled x20;
              W fp32 [256, 64] ~N(0, 0.02); bias ~N(0, 0.01); G = 16; seed 0
  bert_ffn    x bf16 [4096, 768] ~N(0,1), 1% of channels (8) scaled x30;
              W1 [3072, 768], W2 [768, 3072] ~N(0, 0.02); G = 64; seed 1
  gptj_qkv    x bf16 [2048, 4096] = 0.5 * Student-t(nu=4), 8 channels x50;
              W [12288, 4096] = N(0,1) * 0.015 * m_o, m_o log-uniform in
              [0.1, 10] per output row; G = 128; seed 2
  neox_decode x bf16 [16, 6144] ~N(0,1), 0.5% of channels (31) scaled x40;
              W [24576, 6144] ~N(0, 0.01); G = 256; GeLU; seed 3
  ln_sweep    x bf16 [T, H] Student-t(nu=3); seed 100 + point index
  gemm_sweep  x bf16 [M, 8192] Student-t(nu=3); W [8192, 8192] ~N(0, 0.02);
              G = 128; seed 100 + point index
LayerNorm gamma = 1 + 0.1 N(0,1), beta = 0.1 N(0,1), eps = 1e-5 and
bias ~N(0, 0.01) for every workload.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

EPS = 1e-5


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclass
class Activation:
    """An activation matrix as both sides receive it: ``f32`` holds the exact
    values; ``bf16`` holds the bit patterns when the workload is bf16."""
    f32: np.ndarray
    bf16: np.ndarray | None = None

    @property
    def dtype(self) -> str:
        return "bf16" if self.bf16 is not None else "f32"


def _as_act(x: np.ndarray, bf16: bool) -> Activation:
    if not bf16:
        return Activation(np.ascontiguousarray(x, np.float32))
    bits = bf16_bits(x)
    return Activation(bf16_to_f32(bits), bits)


def _outliers(rng, x: np.ndarray, n_ch: int, factor: float, channels=None) -> np.ndarray:
    if channels is None:
        channels = np.sort(rng.permutation(x.shape[1])[:n_ch])
    x[:, channels] *= factor
    return channels


def _ln_params(rng, H):
    gamma = (1.0 + 0.1 * rng.standard_normal(H)).astype(np.float32)
    beta = (0.1 * rng.standard_normal(H)).astype(np.float32)
    return gamma, beta


@dataclass
class Linear:
    W: np.ndarray          # fp32 [N, K]
    bias: np.ndarray       # fp32 [N]
    group_rows: int


@dataclass
class Workload:
    name: str
    x: Activation
    gamma: np.ndarray | None
    beta: np.ndarray | None
    layers: list = field(default_factory=list)
    act: int = 0           # activation of the first linear: 0 none, 1 GeLU
    out: str = "f32"       # output dtype of the last linear
    eps: float = EPS
    outlier_channels: np.ndarray | None = None


def tiny(seed: int = 0) -> Workload:
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((16, 64)).astype(np.float32)
    ch = _outliers(rng, x, 2, 20.0, channels=np.array([3, 41]))
    gamma, beta = _ln_params(rng, 64)
    W = (0.02 * rng.standard_normal((256, 64))).astype(np.float32)
    bias = (0.01 * rng.standard_normal(256)).astype(np.float32)
    return Workload("tiny_w8a8_linear_16x64x256_g16", _as_act(x, False), gamma, beta,
                    [Linear(W, bias, 16)], act=0, out="f32", outlier_channels=ch)


def bert_ffn(seed: int = 1, T: int = 4096) -> Workload:
    rng = np.random.default_rng(seed)
    H, F = 768, 3072
    x = rng.standard_normal((T, H)).astype(np.float32)
    ch = _outliers(rng, x, 8, 30.0)
    gamma, beta = _ln_params(rng, H)
    W1 = (0.02 * rng.standard_normal((F, H))).astype(np.float32)
    b1 = (0.01 * rng.standard_normal(F)).astype(np.float32)
    W2 = (0.02 * rng.standard_normal((H, F))).astype(np.float32)
    b2 = (0.01 * rng.standard_normal(H)).astype(np.float32)
    return Workload(f"bert_base_ffn_block_{T}x768x3072_g64", _as_act(x, True), gamma, beta,
                    [Linear(W1, b1, 64), Linear(W2, b2, 64)], act=1, out="bf16",
                    outlier_channels=ch)


def gptj_qkv(seed: int = 2, T: int = 2048) -> Workload:
    rng = np.random.default_rng(seed)
    H, N = 4096, 12288
    x = (0.5 * rng.standard_t(4.0, size=(T, H))).astype(np.float32)
    ch = _outliers(rng, x, 8, 50.0)
    gamma, beta = _ln_params(rng, H)
    m = np.exp(rng.uniform(np.log(0.1), np.log(10.0), size=N))
    W = (rng.standard_normal((N, H)) * 0.015 * m[:, None]).astype(np.float32)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    return Workload(f"gptj_6b_qkv_{T}x4096x12288_g128", _as_act(x, True), gamma, beta,
                    [Linear(W, bias, 128)], act=0, out="bf16", outlier_channels=ch)


def neox_decode(seed: int = 3, T: int = 16) -> Workload:
    rng = np.random.default_rng(seed)
    H, N = 6144, 24576
    x = rng.standard_normal((T, H)).astype(np.float32)
    ch = _outliers(rng, x, 31, 40.0)
    W = (0.01 * rng.standard_normal((N, H))).astype(np.float32)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    return Workload(f"neox_20b_ffn_up_decode_{T}x6144x24576_g256", _as_act(x, True), None, None,
                    [Linear(W, bias, 256)], act=1, out="bf16", outlier_channels=ch)


LN_SWEEP_T = (1, 64, 1024, 16384, 65536)
LN_SWEEP_H = (1024, 4096, 12288)
GEMM_SWEEP_M = (16, 256, 4096, 16384)


def ln_sweep_point(T: int, H: int, index: int) -> Workload:
    rng = np.random.default_rng(100 + index)
    x = rng.standard_t(3.0, size=(T, H)).astype(np.float32)
    gamma, beta = _ln_params(rng, H)
    return Workload(f"ln_quant_sweep_{T}x{H}", _as_act(x, True), gamma, beta)


def gemm_sweep_point(M: int, index: int, K: int = 8192, N: int = 8192) -> Workload:
    rng = np.random.default_rng(100 + index)
    x = rng.standard_t(3.0, size=(M, K)).astype(np.float32)
    W = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    return Workload(f"gemm_sweep_{M}x{K}x{N}_g128", _as_act(x, True), None, None,
                    [Linear(W, bias, 128)], act=0, out="bf16")


def random_case(seed: int, T: int, K: int, N: int, G: int, dtype: str = "bf16",
                outlier_factor: float = 25.0) -> Workload:
    """Generic ragged-shape case for parity tests."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, K)).astype(np.float32)
    ch = _outliers(rng, x, max(1, K // 100), outlier_factor)
    gamma, beta = _ln_params(rng, K)
    W = (0.02 * rng.standard_normal((N, K))).astype(np.float32)
    bias = (0.01 * rng.standard_normal(N)).astype(np.float32)
    return Workload(f"random_{T}x{K}x{N}_g{G}", _as_act(x, dtype == "bf16"), gamma, beta,
                    [Linear(W, bias, G)], outlier_channels=ch)
