"""CPU oracle for the W8A8 linear hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never imports, links or calls it, and it shares no code with
that path: the arithmetic lives in ``zq_oracle.c`` (plain C loops, compiled
with ``gcc -O2 -ffp-contract=off``), and this module only marshals numpy
arrays and composes the C steps in the order the sources give.

Sources (web pages):
  [ZQ]   "[2022 NeurIPS] ZeroQuant: Efficient and Affordable Post-Training
         Quantization for Large-Scale Transformers" -- token-wise and
         group-wise quantization paragraphs; fused-kernel flowcharts.
  [TS36] "探秘Transformer系列之（36）— 大模型量化方案" -- §1.1.2, §1.2.2.
  [IQ]   "Integer Quantization: Deep Dive" -- quantization formula,
         fake quantization, quantization error.
  [SQ]   "SmoothQuant技术解析：大模型INT8量化的突破与实践" §2.2, §3 and [TS36]
         §1.3 -- per-channel smoothing folded offline into the weights.
  [TS36] §1.1 LLM.int8() -- mixed-precision decomposition of outlier columns.
  [ZQ], [TS36] §1.2.2 group-wise paragraph read along the input axis
         (reading R17 of zq_oracle.c) -- K-axis weight groups.

Every function here is pinned by the ``tests/test_oracle_*.py`` files
against hand-worked examples (``tests/golden/``), closed forms, invariants
and library routines; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zq_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libzqoracle.so")

ACT_NONE = 0
ACT_GELU = 1


def build(force: bool = False) -> str:
    """Compile the C oracle to ``oracle/_build/libzqoracle.so`` (no GPU)."""
    os.makedirs(os.path.dirname(_LIB), exist_ok=True)
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P, I64, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
        sig = {
            "zqo_quantize_span": [P, I64, P, P],
            "zqo_quantize_weights": [P, I64, I64, I64, P, P],
            "zqo_quantize_rows": [P, I64, I64, P, P],
            "zqo_layernorm": [P, I64, I64, P, P, F, P],
            "zqo_bias_act": [P, I64, I64, P, ctypes.c_int, P],
            "zqo_gemm_i32": [P, I64, I64, P, I64, P],
            "zqo_dequant": [P, I64, I64, P, P, I64, P, ctypes.c_int, P],
            "zqo_channel_absmax": [P, I64, I64, P],
            "zqo_weight_col_absmax": [P, I64, I64, P],
            "zqo_smooth_factors": [P, P, I64, F, P],
            "zqo_smooth_fold": [P, I64, I64, P, P, P, P, P, P],
            "zqo_outlier_product": [P, I64, I64, P, I64, P, I64, P],
            "zqo_dequant_add": [P, I64, I64, P, P, I64, P, P, ctypes.c_int, P],
            "zqo_quantize_weights_kgroups": [P, I64, I64, I64, P, P],
            "zqo_linear_kgroups": [P, I64, I64, P, I64, I64, P, P, P, ctypes.c_int, P],
        }
        for name, args in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        lib.zqo_outlier_columns.argtypes = [P, I64, F, P, I64]
        lib.zqo_outlier_columns.restype = I64
        _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _chk(rc, what):
    if rc == 2:
        raise OracleError(f"{what}: int32 accumulator overflow")
    if rc != 0:
        raise OracleError(f"{what}: bad argument (status {rc})")


def quantize_span(v):
    """Absmax symmetric quantization of one vector ([TS36] §1.1.2).
    Returns (int8 codes, fp32 scale)."""
    v, pv = _c(v, np.float32)
    q = np.empty(v.shape, np.int8)
    s = np.zeros(1, np.float32)
    _chk(_L().zqo_quantize_span(pv, v.size, q.ctypes.data, s.ctypes.data), "quantize_span")
    return q, s[0]


def quantize_weights(W, group_rows):
    """Group-wise weight quantization ([ZQ]; [TS36] §1.2.2): W fp32 [N, K]
    -> (Wq int8 [N, K], s_grp fp32 [N / group_rows])."""
    W, pw = _c(W, np.float32)
    N, K = W.shape
    Wq = np.empty((N, K), np.int8)
    s = np.empty(N // group_rows if group_rows > 0 else 0, np.float32)
    _chk(_L().zqo_quantize_weights(pw, N, K, group_rows, Wq.ctypes.data, s.ctypes.data),
         "quantize_weights")
    return Wq, s


def quantize_rows(Y):
    """Per-token (row) quantization of fp32 Y [T, H] -> (q int8, s_tok fp32 [T])."""
    Y, py = _c(Y, np.float32)
    T, H = Y.shape
    q = np.empty((T, H), np.int8)
    s = np.empty(T, np.float32)
    _chk(_L().zqo_quantize_rows(py, T, H, q.ctypes.data, s.ctypes.data), "quantize_rows")
    return q, s


def layernorm(x, gamma, beta, eps):
    """LayerNorm in double, rounded to fp32 (biased variance, eps inside sqrt)."""
    x, px = _c(x, np.float32)
    g, pg = _c(gamma, np.float32)
    b, pb = _c(beta, np.float32)
    T, H = x.shape
    y = np.empty((T, H), np.float32)
    _chk(_L().zqo_layernorm(px, T, H, pg, pb, float(eps), y.ctypes.data), "layernorm")
    return y


def bias_act(x, bias=None, act=ACT_NONE):
    """y = act(x + bias) in double, rounded to fp32 (act: identity or exact GeLU)."""
    x, px = _c(x, np.float32)
    T, H = x.shape
    pb = None
    if bias is not None:
        bias, pb = _c(bias, np.float32)
    y = np.empty((T, H), np.float32)
    _chk(_L().zqo_bias_act(px, T, H, pb, int(act), y.ctypes.data), "bias_act")
    return y


def gemm_i32(xq, Wq):
    """acc[t, o] = sum_k xq[t, k] * Wq[o, k], exact, int32 result."""
    xq, px = _c(xq, np.int8)
    Wq, pw = _c(Wq, np.int8)
    T, K = xq.shape
    N, K2 = Wq.shape
    if K != K2:
        raise OracleError("gemm_i32: K mismatch")
    acc = np.empty((T, N), np.int32)
    _chk(_L().zqo_gemm_i32(px, T, K, pw, N, acc.ctypes.data), "gemm_i32")
    return acc


def dequant(acc, s_tok, s_grp, group_rows, bias=None, act=ACT_NONE):
    """y = act(s_tok[t] * s_grp[o // G] * acc[t, o] + bias[o]) in double -> fp32."""
    acc, pa = _c(acc, np.int32)
    st, ps = _c(s_tok, np.float32)
    sg, pg = _c(s_grp, np.float32)
    T, N = acc.shape
    pb = None
    if bias is not None:
        bias, pb = _c(bias, np.float32)
    y = np.empty((T, N), np.float32)
    _chk(_L().zqo_dequant(pa, T, N, ps, pg, group_rows, pb, int(act), y.ctypes.data),
         "dequant")
    return y


def channel_absmax(a, amax=None):
    """Running per-channel absmax of an activation a [T, H] ([SQ] §3 calibration)."""
    a, pa = _c(a, np.float32)
    T, H = a.shape
    out = np.zeros(H, np.float32) if amax is None else np.array(amax, np.float32, copy=True)
    _chk(_L().zqo_channel_absmax(pa, T, H, out.ctypes.data), "channel_absmax")
    return out


def weight_col_absmax(W):
    """Per input channel absmax of W [N, K]: max over the N output rows."""
    W, pw = _c(W, np.float32)
    N, K = W.shape
    out = np.empty(K, np.float32)
    _chk(_L().zqo_weight_col_absmax(pw, N, K, out.ctypes.data), "weight_col_absmax")
    return out


def smooth_factors(amax, wmax, alpha=0.5):
    """s_j = amax_j^alpha / wmax_j^(1-alpha) (reading R14 of zq_oracle.c);
    alpha is taken as an fp32 value, as the library's interface passes it."""
    a, pa = _c(amax, np.float32)
    w, pw = _c(wmax, np.float32)
    s = np.empty(a.size, np.float32)
    _chk(_L().zqo_smooth_factors(pa, pw, a.size, float(alpha), s.ctypes.data), "smooth_factors")
    return s


def smooth_fold(W, s, gamma=None, beta=None):
    """W' = W diag(s) per input channel; gamma' = gamma / s, beta' = beta / s."""
    W, pw = _c(W, np.float32)
    s_, ps = _c(s, np.float32)
    N, K = W.shape
    Wo = np.empty((N, K), np.float32)
    pg = pb = None
    go = bo = None
    if gamma is not None:
        gamma, pg = _c(gamma, np.float32)
        go = np.empty(K, np.float32)
    if beta is not None:
        beta, pb = _c(beta, np.float32)
        bo = np.empty(K, np.float32)
    _chk(_L().zqo_smooth_fold(pw, N, K, pg, pb, ps, Wo.ctypes.data,
                              None if go is None else go.ctypes.data,
                              None if bo is None else bo.ctypes.data), "smooth_fold")
    return Wo, go, bo


# ---- compositions, in the order of the fused flowcharts of [ZQ] ----------

def ln_quant(x, gamma, beta, eps):
    """Fused "LN + Quantize": LayerNorm, then per-token quantization."""
    return quantize_rows(layernorm(x, gamma, beta, eps))


def act_quant(x, bias=None, act=ACT_NONE):
    """Fused "GeLU + Quantize" (or plain token quantization when act is none)."""
    return quantize_rows(bias_act(x, bias, act))


def linear(xq, s_tok, Wq, s_grp, group_rows, bias=None, act=ACT_NONE):
    """Fused "GEMM + DeQuantize": int32 GEMM then the dequant epilogue, fp32 out."""
    return dequant(gemm_i32(xq, Wq), s_tok, s_grp, group_rows, bias, act)


def linear_requant(xq, s_tok, Wq, s_grp, group_rows, bias=None, act=ACT_GELU):
    """GEMM + DeQuantize + act, then per-token quantization for the next layer."""
    return quantize_rows(linear(xq, s_tok, Wq, s_grp, group_rows, bias, act))


def ffn_block(x, gamma, beta, eps, W1q, s1, b1, W2q, s2, b2, group_rows):
    """Transformer FFN as the fused kernels run it:
    LN+quant -> GEMM1+dequant+bias+GeLU+requant -> GEMM2+dequant+bias (fp32).
    Returns the fp32 output and the intermediate (q1, s_tok1, q2, s_tok2)."""
    q1, st1 = ln_quant(x, gamma, beta, eps)
    q2, st2 = linear_requant(q1, st1, W1q, s1, group_rows, b1, ACT_GELU)
    y = linear(q2, st2, W2q, s2, group_rows, b2, ACT_NONE)
    return y, (q1, st1, q2, st2)


def smooth_ln_linear(calib_batches, gamma, beta, eps, W, alpha=0.5):
    """SmoothQuant offline step for a linear fed by a LayerNorm ([TS36] §1.3,
    [SQ] §3): calibrate the per-channel absmax of the LayerNorm output over
    the batches, derive s, fold diag(s)^-1 into gamma/beta and diag(s) into
    W.  Returns (W', gamma', beta', s, activation absmax)."""
    amax = None
    for xb in calib_batches:
        amax = channel_absmax(layernorm(xb, gamma, beta, eps), amax)
    s = smooth_factors(amax, weight_col_absmax(W), alpha)
    Wo, go, bo = smooth_fold(W, s, gamma, beta)
    return Wo, go, bo, s, amax


# ---- LLM.int8() mixed-precision decomposition ([TS36] §1.1, reading R16) ---

LLM_INT8_ALPHA = 6.0


def outlier_columns(amax, threshold=LLM_INT8_ALPHA, max_o=8):
    """Columns with amax >= threshold, ascending; returns (first max_o of them, total count)."""
    a, pa = _c(amax, np.float32)
    idx = np.zeros(max(max_o, 1), np.int32)
    n = _L().zqo_outlier_columns(pa, a.size, float(threshold), idx.ctypes.data, int(max_o))
    if n < 0:
        raise OracleError("outlier_columns: bad argument")
    return idx[:min(n, max_o)].copy(), int(n)


def outlier_product(a, W, idx):
    """sum over the listed columns j of fp16(a[t, j]) * fp16(W[o, j]), in float64."""
    a, pa = _c(a, np.float32)
    W, pw = _c(W, np.float32)
    ix, pi = _c(idx, np.int32)
    T, K = a.shape
    N = W.shape[0]
    out = np.empty((T, N), np.float64)
    _chk(_L().zqo_outlier_product(pa, T, K, pw, N, pi if ix.size else None, ix.size, out.ctypes.data),
         "outlier_product")
    return out


def dequant_add(acc, s_tok, s_grp, group_rows, add=None, bias=None, act=ACT_NONE):
    """y = act(s_tok s_grp acc + add + bias) in double -> fp32."""
    acc, pa = _c(acc, np.int32)
    st, ps = _c(s_tok, np.float32)
    sg, pg = _c(s_grp, np.float32)
    T, N = acc.shape
    pad = pb = None
    if add is not None:
        add, pad = _c(add, np.float64)
    if bias is not None:
        bias, pb = _c(bias, np.float32)
    y = np.empty((T, N), np.float32)
    _chk(_L().zqo_dequant_add(pa, T, N, ps, pg, group_rows, pad, pb, int(act), y.ctypes.data), "dequant_add")
    return y


def int8_decomposed_ln_linear(x, gamma, beta, eps, W, Wq, s_grp, group_rows, bias=None, act=ACT_NONE,
                              threshold=LLM_INT8_ALPHA, max_o=8):
    """LLM.int8() on a LayerNorm-fed linear: detect the outlier columns of the
    LayerNorm output over the batch, quantize the other columns per token
    (the outlier columns contribute zero codes), run the INT8 GEMM with the
    group-quantized weights, add the fp16 outlier product, then bias and
    activation.  Returns (y fp32, outlier columns, total outlier count)."""
    a = layernorm(x, gamma, beta, eps)
    idx, n = outlier_columns(channel_absmax(a), threshold, max_o)
    a_in = a.copy()
    a_in[:, idx] = 0.0
    xq, st = quantize_rows(a_in)
    add = outlier_product(a, W, idx)
    y = dequant_add(gemm_i32(xq, Wq), st, s_grp, group_rows, add, bias, act)
    return y, idx, n


# ---- K-axis weight groups ([ZQ], [TS36] §1.2.2, reading R17) ---------------

def quantize_weights_kgroups(W, group_cols):
    """Group-wise weight quantization along the input axis: W fp32 [N, K] ->
    (Wq int8 [N, K], s_w fp32 [N, K / group_cols]); group (o, j) is row o,
    columns j*group_cols .. (j+1)*group_cols - 1."""
    W, pw = _c(W, np.float32)
    N, K = W.shape
    Wq = np.empty((N, K), np.int8)
    s = np.empty((N, K // group_cols if group_cols > 0 else 0), np.float32)
    _chk(_L().zqo_quantize_weights_kgroups(pw, N, K, group_cols, Wq.ctypes.data, s.ctypes.data),
         "quantize_weights_kgroups")
    return Wq, s


def linear_kgroups(xq, s_tok, Wq, s_w, group_cols, bias=None, act=ACT_NONE):
    """y = act(s_tok[t] * sum_j s_w[o, j] * acc_j[t, o] + bias[o]) in double -> fp32,
    acc_j the exact integer product over the columns of group j."""
    xq, px = _c(xq, np.int8)
    Wq, pw = _c(Wq, np.int8)
    st, ps = _c(s_tok, np.float32)
    sw, pg = _c(s_w, np.float32)
    T, K = xq.shape
    N, K2 = Wq.shape
    if K != K2 or sw.shape != (N, K // group_cols):
        raise OracleError("linear_kgroups: shape mismatch")
    pb = None
    if bias is not None:
        bias, pb = _c(bias, np.float32)
    y = np.empty((T, N), np.float32)
    _chk(_L().zqo_linear_kgroups(px, T, K, pw, N, group_cols, ps, pg, pb, int(act), y.ctypes.data),
         "linear_kgroups")
    return y


def ln_linear_kgroups(x, gamma, beta, eps, Wq, s_w, group_cols, bias=None, act=ACT_NONE):
    """LN + per-token quantization, then the K-group linear (fp32 out)."""
    xq, st = ln_quant(x, gamma, beta, eps)
    return linear_kgroups(xq, st, Wq, s_w, group_cols, bias, act)

