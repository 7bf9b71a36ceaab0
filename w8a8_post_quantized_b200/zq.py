"""Python binding of the C ABI in ``include/zq.h`` (``libzq.so``).

Argument marshalling only: every step of the path runs in the library's
sm_100a kernels.  torch supplies device memory and streams.  The functions
carry the C names; each validates nothing the library does not validate
itself, allocates outputs with ``torch.empty`` when they are not given, and
raises :class:`ZQError` on a non-zero status.

There is no fallback: importing this module fails loudly when ``libzq.so``
has not been built (``python -m w8a8_post_quantized_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libzq.so")

# ---- enums, mirroring include/zq.h ---------------------------------------
ZQ_OK, ZQ_ERR_NULL, ZQ_ERR_SHAPE, ZQ_ERR_ALIGN, ZQ_ERR_OVERFLOW = 0, 1, 2, 3, 4
ZQ_ERR_DTYPE, ZQ_ERR_CUDA, ZQ_ERR_TIMEOUT, ZQ_ERR_WORKSPACE, ZQ_ERR_DEVICE = 5, 6, 7, 8, 9
ZQ_ERR_SCRATCH = 10
ZQ_NOALLOC_SCRATCH_BYTES = 64 << 20
ZQ_F32, ZQ_BF16 = 0, 1
ZQ_ACT_NONE, ZQ_ACT_GELU = 0, 1
ZQ_OUT_F32, ZQ_OUT_BF16, ZQ_OUT_I8_REQUANT, ZQ_OUT_I32_RAW = 0, 1, 2, 3
ZQ_MAX_K = 133144
ZQ_MAX_H = 65536

EXPORTED = (
    "zq_quantize_weights", "zq_ln_quant", "zq_act_quant", "zq_w8a8_linear_workspace",
    "zq_w8a8_linear", "zq_linear_block_workspace", "zq_linear_block", "zq_device_status",
    "zq_status_string", "zq_last_cuda_error", "zq_version", "zq_launch_count",
    "zq_w8a8_linear_requant_noalloc", "zq_smooth_calibrate", "zq_smooth_weights",
    "zq_watchdog_selftest", "zq_llmint8_select", "zq_llmint8_outlier_act", "zq_llmint8_outlier_weights",
    "zq_w8a8_linear_llmint8", "zq_quantize_weights_kgroups", "zq_w8a8_linear_kgroups",
)
ZQ_LLMINT8_MAX_OUTLIERS = 8


class ZQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().zq_status_string(status).decode()
        if status == ZQ_ERR_CUDA:
            msg += f" ({lib().zq_last_cuda_error().decode()})"
        super().__init__(f"{where}: status {status}: {msg}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library, with argument types declared for every entry point."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libzq.so not built at {_LIB_PATH}; run "
                          "`python -m w8a8_post_quantized_b200.build` (needs nvcc)")
    L = ctypes.CDLL(_LIB_PATH)
    P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    sigs = {
        "zq_quantize_weights": (I, [P, I64, I64, I64, P, P, P]),
        "zq_ln_quant": (I, [P, I, I64, I64, P, P, F, P, P, P]),
        "zq_act_quant": (I, [P, I, I64, I64, P, I, P, P, P]),
        "zq_w8a8_linear_workspace": (SZ, [I64, I64, I64, I]),
        "zq_w8a8_linear": (I, [P, P, I64, I64, P, P, I64, I64, P, I, I, P, P, P, SZ, P]),
        "zq_linear_block_workspace": (SZ, [I64, I64, I64, I]),
        "zq_linear_block": (I, [P, I, I64, I64, P, P, F, P, P, I64, I64, P, I, I, P, P, P, SZ, P]),
        "zq_device_status": (I, [P]),
        "zq_status_string": (ctypes.c_char_p, [I]),
        "zq_last_cuda_error": (ctypes.c_char_p, []),
        "zq_version": (I, []),
        "zq_launch_count": (ctypes.c_uint64, []),
        "zq_w8a8_linear_requant_noalloc": (I, [P, P, I64, I64, P, P, I64, I64, P, I, P, P, P]),
        "zq_smooth_calibrate": (I, [P, I, I64, I64, P, P, F, P, P]),
        "zq_smooth_weights": (I, [P, I64, I64, P, F, P, P, P, P, P, P, P]),
        "zq_watchdog_selftest": (I, [P]),
        "zq_llmint8_select": (I, [P, I64, F, P, P, P, P, P, P, P]),
        "zq_llmint8_outlier_act": (I, [P, I, I64, I64, P, P, F, P, P, P, P]),
        "zq_llmint8_outlier_weights": (I, [P, I64, I64, P, P, P, P]),
        "zq_w8a8_linear_llmint8": (I, [P, P, I64, I64, P, P, I64, I64, P, I, I, P, P, P, P]),
        "zq_quantize_weights_kgroups": (I, [P, I64, I64, I64, P, P, P]),
        "zq_w8a8_linear_kgroups": (I, [P, P, I64, I64, P, P, I64, I64, P, I, I, P, P]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(x: torch.Tensor) -> int:
    if x.dtype == torch.bfloat16:
        return ZQ_BF16
    if x.dtype == torch.float32:
        return ZQ_F32
    raise TypeError(f"activation dtype {x.dtype} not supported (bf16 or fp32)")


def _check(rc: int, where: str):
    if rc != ZQ_OK:
        raise ZQError(rc, where)


def _out_dtype(out_kind: int):
    return {ZQ_OUT_F32: torch.float32, ZQ_OUT_BF16: torch.bfloat16,
            ZQ_OUT_I8_REQUANT: torch.int8, ZQ_OUT_I32_RAW: torch.int32}[out_kind]


# ---- entry points ---------------------------------------------------------

def zq_quantize_weights(W, group_rows, Wq=None, s_grp=None, stream=None):
    N, K = W.shape
    Wq = torch.empty((N, K), dtype=torch.int8, device=W.device) if Wq is None else Wq
    s_grp = (torch.empty(N // max(group_rows, 1), dtype=torch.float32, device=W.device)
             if s_grp is None else s_grp)
    _check(lib().zq_quantize_weights(_p(W), N, K, group_rows, _p(Wq), _p(s_grp), _s(stream)),
           "zq_quantize_weights")
    return Wq, s_grp


def zq_ln_quant(x, gamma, beta, eps, q=None, s_tok=None, stream=None):
    T, H = x.shape
    q = torch.empty((T, H), dtype=torch.int8, device=x.device) if q is None else q
    s_tok = torch.empty(T, dtype=torch.float32, device=x.device) if s_tok is None else s_tok
    _check(lib().zq_ln_quant(_p(x), _dtype_code(x), T, H, _p(gamma), _p(beta), float(eps),
                             _p(q), _p(s_tok), _s(stream)), "zq_ln_quant")
    return q, s_tok


def zq_smooth_calibrate(x, gamma=None, beta=None, eps=1e-5, amax=None, stream=None):
    """Running per-channel absmax of LayerNorm(x) (or x without gamma); pass
    the returned amax back in for the next calibration batch."""
    T, H = x.shape
    amax = torch.zeros(H, dtype=torch.float32, device=x.device) if amax is None else amax
    _check(lib().zq_smooth_calibrate(_p(x), _dtype_code(x), T, H, _p(gamma), _p(beta), float(eps),
                                     _p(amax), _s(stream)), "zq_smooth_calibrate")
    return amax


def zq_smooth_weights(W, amax, alpha=0.5, gamma=None, beta=None, W_out=None, gamma_out=None,
                      beta_out=None, s=None, stream=None):
    """SmoothQuant factors and fold: returns (W_out, gamma_out, beta_out, s)."""
    N, K = W.shape
    W_out = torch.empty_like(W) if W_out is None else W_out
    if gamma is not None and gamma_out is None:
        gamma_out = torch.empty_like(gamma)
    if beta is not None and beta_out is None:
        beta_out = torch.empty_like(beta)
    s = torch.empty(K, dtype=torch.float32, device=W.device) if s is None else s
    _check(lib().zq_smooth_weights(_p(W), N, K, _p(amax), float(alpha), _p(gamma), _p(beta),
                                   _p(W_out), _p(gamma_out), _p(beta_out), _p(s), _s(stream)),
           "zq_smooth_weights")
    return W_out, gamma_out, beta_out, s


def zq_llmint8_select(amax, gamma, beta=None, threshold=6.0, stream=None):
    """LLM.int8() outlier columns: returns (idx [8] int32, count [1] int32,
    gamma and beta zeroed on the decomposed columns)."""
    K = amax.numel()
    dev = amax.device
    idx = torch.empty(ZQ_LLMINT8_MAX_OUTLIERS, dtype=torch.int32, device=dev)
    count = torch.empty(1, dtype=torch.int32, device=dev)
    gm = torch.empty(K, dtype=torch.float32, device=dev)
    bm = torch.empty(K, dtype=torch.float32, device=dev)
    _check(lib().zq_llmint8_select(_p(amax), K, float(threshold), _p(gamma), _p(beta), _p(idx), _p(count),
                                   _p(gm), _p(bm), _s(stream)), "zq_llmint8_select")
    return idx, count, gm, bm


def zq_llmint8_outlier_act(x, gamma, beta, eps, idx, count, stream=None):
    """The decomposed columns of LayerNorm(x) as fp16 [T, 8]."""
    T, K = x.shape
    xo = torch.empty((T, ZQ_LLMINT8_MAX_OUTLIERS), dtype=torch.float16, device=x.device)
    _check(lib().zq_llmint8_outlier_act(_p(x), _dtype_code(x), T, K, _p(gamma), _p(beta), float(eps), _p(idx),
                                        _p(count), _p(xo), _s(stream)), "zq_llmint8_outlier_act")
    return xo


def zq_llmint8_outlier_weights(W, idx, count, stream=None):
    """The decomposed columns of the fp32 weights as fp16 [N, 8]."""
    N, K = W.shape
    wo = torch.empty((N, ZQ_LLMINT8_MAX_OUTLIERS), dtype=torch.float16, device=W.device)
    _check(lib().zq_llmint8_outlier_weights(_p(W), N, K, _p(idx), _p(count), _p(wo), _s(stream)),
           "zq_llmint8_outlier_weights")
    return wo


def zq_w8a8_linear_llmint8(xq, s_tok, Wq, s_grp, group_rows, xo, wo, bias=None, act=ZQ_ACT_NONE,
                           out_kind=ZQ_OUT_BF16, y=None, stream=None):
    """W8A8 linear plus the fp16 outlier product (before bias and activation)."""
    T, K = xq.shape
    N = Wq.shape[0]
    y = torch.empty((T, N), dtype=_out_dtype(out_kind), device=xq.device) if y is None else y
    _check(lib().zq_w8a8_linear_llmint8(_p(xq), _p(s_tok), T, K, _p(Wq), _p(s_grp), N, group_rows, _p(bias),
                                        int(act), int(out_kind), _p(xo), _p(wo), _p(y), _s(stream)),
           "zq_w8a8_linear_llmint8")
    return y


def zq_quantize_weights_kgroups(W, group_cols, Wq=None, s_w=None, stream=None):
    """K-axis groups: returns Wq int8 [N, K] and the group-major scales s_w
    fp32 [K / group_cols, N]."""
    N, K = W.shape
    Wq = torch.empty((N, K), dtype=torch.int8, device=W.device) if Wq is None else Wq
    s_w = (torch.empty((K // max(group_cols, 1), N), dtype=torch.float32, device=W.device)
           if s_w is None else s_w)
    _check(lib().zq_quantize_weights_kgroups(_p(W), N, K, group_cols, _p(Wq), _p(s_w), _s(stream)),
           "zq_quantize_weights_kgroups")
    return Wq, s_w


def zq_w8a8_linear_kgroups(xq, s_tok, Wq, s_w, group_cols, bias=None, act=ZQ_ACT_NONE,
                           out_kind=ZQ_OUT_BF16, y=None, stream=None):
    """W8A8 linear with K-axis weight groups (s_w group-major [K / group_cols, N])."""
    T, K = xq.shape
    N = Wq.shape[0]
    y = torch.empty((T, N), dtype=_out_dtype(out_kind), device=xq.device) if y is None else y
    _check(lib().zq_w8a8_linear_kgroups(_p(xq), _p(s_tok), T, K, _p(Wq), _p(s_w), N, group_cols, _p(bias),
                                        int(act), int(out_kind), _p(y), _s(stream)),
           "zq_w8a8_linear_kgroups")
    return y


def zq_act_quant(x, bias=None, act=ZQ_ACT_NONE, q=None, s_tok=None, stream=None):
    T, H = x.shape
    q = torch.empty((T, H), dtype=torch.int8, device=x.device) if q is None else q
    s_tok = torch.empty(T, dtype=torch.float32, device=x.device) if s_tok is None else s_tok
    _check(lib().zq_act_quant(_p(x), _dtype_code(x), T, H, _p(bias), int(act), _p(q), _p(s_tok),
                              _s(stream)), "zq_act_quant")
    return q, s_tok


def zq_w8a8_linear_workspace(T, K, N, out_kind) -> int:
    return int(lib().zq_w8a8_linear_workspace(T, K, N, out_kind))


def zq_w8a8_linear(xq, s_tok, Wq, s_grp, group_rows, bias=None, act=ZQ_ACT_NONE,
                   out_kind=ZQ_OUT_BF16, y=None, s_tok_out=None, workspace=None, stream=None):
    T, K = xq.shape
    N = Wq.shape[0]
    dev = xq.device
    y = torch.empty((T, N), dtype=_out_dtype(out_kind), device=dev) if y is None else y
    if out_kind == ZQ_OUT_I8_REQUANT and s_tok_out is None:
        s_tok_out = torch.empty(T, dtype=torch.float32, device=dev)
    need = zq_w8a8_linear_workspace(T, K, N, out_kind)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().zq_w8a8_linear(_p(xq), _p(s_tok), T, K, _p(Wq), _p(s_grp), N, group_rows,
                                _p(bias), int(act), int(out_kind), _p(y), _p(s_tok_out),
                                _p(workspace), ws_bytes, _s(stream)), "zq_w8a8_linear")
    return (y, s_tok_out) if out_kind == ZQ_OUT_I8_REQUANT else y


def zq_linear_block_workspace(T, K, N, out_kind) -> int:
    return int(lib().zq_linear_block_workspace(T, K, N, out_kind))


def zq_linear_block(x, gamma, beta, eps, Wq, s_grp, group_rows, bias=None, act=ZQ_ACT_NONE,
                    out_kind=ZQ_OUT_BF16, y=None, s_tok_out=None, workspace=None, stream=None):
    T, K = x.shape
    N = Wq.shape[0]
    dev = x.device
    y = torch.empty((T, N), dtype=_out_dtype(out_kind), device=dev) if y is None else y
    if out_kind == ZQ_OUT_I8_REQUANT and s_tok_out is None:
        s_tok_out = torch.empty(T, dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(zq_linear_block_workspace(T, K, N, out_kind), dtype=torch.uint8,
                                device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib().zq_linear_block(_p(x), _dtype_code(x), T, K, _p(gamma), _p(beta), float(eps),
                                 _p(Wq), _p(s_grp), N, group_rows, _p(bias), int(act),
                                 int(out_kind), _p(y), _p(s_tok_out), _p(workspace), ws_bytes,
                                 _s(stream)), "zq_linear_block")
    return (y, s_tok_out) if out_kind == ZQ_OUT_I8_REQUANT else y


def zq_w8a8_linear_requant_noalloc(xq, s_tok, Wq, s_grp, group_rows, bias=None,
                                   act=ZQ_ACT_GELU, y=None, s_tok_out=None, stream=None):
    """Requantizing linear that uses the library's fixed scratch array instead of
    a workspace (for callers that cannot allocate device memory).  The outputs
    must be passed in by such callers; they are allocated here only as a
    convenience for callers that can."""
    T, K = xq.shape
    N = Wq.shape[0]
    y = torch.empty((T, N), dtype=torch.int8, device=xq.device) if y is None else y
    s_tok_out = torch.empty(T, dtype=torch.float32, device=xq.device) if s_tok_out is None else s_tok_out
    _check(lib().zq_w8a8_linear_requant_noalloc(_p(xq), _p(s_tok), T, K, _p(Wq), _p(s_grp), N,
                                                group_rows, _p(bias), int(act), _p(y),
                                                _p(s_tok_out), _s(stream)),
           "zq_w8a8_linear_requant_noalloc")
    return y, s_tok_out


def zq_device_status(stream=None):
    _check(lib().zq_device_status(_s(stream)), "zq_device_status")


def zq_watchdog_selftest(stream=None):
    """Enqueue a kernel whose bounded wait expires (about 2 s); the next
    zq_device_status() raises ZQError with ZQ_ERR_TIMEOUT."""
    _check(lib().zq_watchdog_selftest(_s(stream)), "zq_watchdog_selftest")


def zq_version() -> int:
    return int(lib().zq_version())


def zq_launch_count() -> int:
    return int(lib().zq_launch_count())
