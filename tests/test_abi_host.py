"""C-ABI checks that need no GPU.

* the library loads and exports every function ``include/zq.h`` declares;
* every invalid argument is rejected on the host with its documented status
  before anything reaches CUDA.  The pointers used here are fake addresses:
  validation fails first, so they are never dereferenced.  No call with
  valid arguments is made (that would launch work).
"""
import ctypes
import os
import re

import pytest

from w8a8_post_quantized_b200 import zq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "zq.h")

A16 = 0x7F0000000000          # 16-byte aligned fake device address
A16b = 0x7F0000100000
A16c = 0x7F0000200000
MIS = 0x7F0000000001          # misaligned


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("zq_quantize_weights", "zq_ln_quant", "zq_act_quant", "zq_w8a8_linear",
                     "zq_linear_block"):
        assert required in names


def test_library_exports_every_declared_symbol():
    L = zq.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    assert set(declared_functions()) == set(zq.EXPORTED)


def test_status_strings_and_version():
    L = zq.lib()
    for s in range(0, 10):
        txt = L.zq_status_string(s)
        assert txt and txt.decode()
    assert L.zq_status_string(12345).decode() == "unknown status"
    assert zq.zq_version() >= 100
    assert zq.lib().zq_w8a8_linear_workspace(4096, 768, 3072, zq.ZQ_OUT_BF16) == 0
    # at most 64 tokens: the fp32 output and the absmax words
    assert zq.lib().zq_w8a8_linear_workspace(64, 768, 3072, zq.ZQ_OUT_I8_REQUANT) >= 64 * 3072 * 4 + 64 * 4


def test_requant_workspace_without_a_device():
    """With no usable device the query cannot tell whether the fused kernels
    apply and asks for the scratch route's size (fp32 output + absmax words)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert zq.lib().zq_w8a8_linear_workspace(4096, 768, 3072, zq.ZQ_OUT_I8_REQUANT) >= 4096 * 3072 * 4 + 4096 * 4


def _lin(**kw):
    a = dict(xq=A16, s_tok=A16b, T=64, K=128, Wq=A16c, s_grp=A16b, N=256, G=16, bias=None,
             act=0, out=zq.ZQ_OUT_BF16, y=A16, s_out=None, ws=None, ws_bytes=0, stream=None)
    a.update(kw)
    return zq.lib().zq_w8a8_linear(a["xq"], a["s_tok"], a["T"], a["K"], a["Wq"], a["s_grp"], a["N"],
                                   a["G"], a["bias"], a["act"], a["out"], a["y"], a["s_out"],
                                   a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(xq=None), zq.ZQ_ERR_NULL),
    (dict(Wq=None), zq.ZQ_ERR_NULL),
    (dict(y=None), zq.ZQ_ERR_NULL),
    (dict(s_grp=None), zq.ZQ_ERR_NULL),
    (dict(out=zq.ZQ_OUT_I8_REQUANT, s_out=None), zq.ZQ_ERR_NULL),
    (dict(T=0), zq.ZQ_ERR_SHAPE),
    (dict(K=-16), zq.ZQ_ERR_SHAPE),
    (dict(K=120), zq.ZQ_ERR_SHAPE),            # K % 16
    (dict(N=250, G=10), zq.ZQ_ERR_SHAPE),      # N % 16
    (dict(N=256, G=48), zq.ZQ_ERR_SHAPE),      # N % G
    (dict(G=0), zq.ZQ_ERR_SHAPE),
    (dict(K=zq.ZQ_MAX_K + 16 - (zq.ZQ_MAX_K % 16)), zq.ZQ_ERR_OVERFLOW),
    (dict(xq=MIS), zq.ZQ_ERR_ALIGN),
    (dict(Wq=MIS), zq.ZQ_ERR_ALIGN),
    (dict(y=MIS), zq.ZQ_ERR_ALIGN),
    (dict(s_tok=A16 + 2), zq.ZQ_ERR_ALIGN),
    (dict(out=7), zq.ZQ_ERR_DTYPE),
    (dict(act=3), zq.ZQ_ERR_DTYPE),
    (dict(out=zq.ZQ_OUT_I32_RAW, act=zq.ZQ_ACT_GELU), zq.ZQ_ERR_DTYPE),
    (dict(out=zq.ZQ_OUT_I32_RAW, bias=A16), zq.ZQ_ERR_DTYPE),
    (dict(out=zq.ZQ_OUT_I8_REQUANT, s_out=A16b, ws=None, ws_bytes=0), zq.ZQ_ERR_WORKSPACE),
    (dict(out=zq.ZQ_OUT_I8_REQUANT, s_out=A16b, ws=A16c, ws_bytes=100), zq.ZQ_ERR_WORKSPACE),
    # the optional workspace of the other kinds, when given, is 16-byte aligned
    (dict(T=16, out=zq.ZQ_OUT_BF16, ws=MIS, ws_bytes=1 << 20), zq.ZQ_ERR_ALIGN),
    (dict(T=16, out=zq.ZQ_OUT_I32_RAW, ws=A16c + 8, ws_bytes=1 << 20), zq.ZQ_ERR_ALIGN),
])
def test_linear_rejects_bad_arguments_on_host(kw, status):
    assert _lin(**kw) == status


def test_optional_workspace_without_a_device():
    """The few-token even split needs the SM count; with no usable device the
    query offers no workspace for the non-requantizing kinds (a call then
    takes the split-K clusters), whatever the shape."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    for T, K, N in [(16, 6144, 24576), (1, 128, 16), (64, 4096, 65536), (65, 6144, 24576)]:
        for kind in (zq.ZQ_OUT_F32, zq.ZQ_OUT_BF16, zq.ZQ_OUT_I32_RAW):
            assert zq.lib().zq_w8a8_linear_workspace(T, K, N, kind) == 0


def test_max_k_is_the_int32_bound():
    assert zq.ZQ_MAX_K == (2 ** 31 - 1) // (127 * 127)
    assert zq.ZQ_MAX_K % 16 == 8       # so the largest legal K is ZQ_MAX_K - 8


@pytest.mark.parametrize("call,status", [
    (lambda L: L.zq_ln_quant(None, 1, 4, 64, A16, A16, 1e-5, A16, A16, None), zq.ZQ_ERR_NULL),
    (lambda L: L.zq_ln_quant(A16, 1, 4, 64, None, A16, 1e-5, A16, A16, None), zq.ZQ_ERR_NULL),
    (lambda L: L.zq_ln_quant(A16, 1, 4, 60, A16, A16, 1e-5, A16, A16, None), zq.ZQ_ERR_SHAPE),
    (lambda L: L.zq_ln_quant(A16, 1, 0, 64, A16, A16, 1e-5, A16, A16, None), zq.ZQ_ERR_SHAPE),
    (lambda L: L.zq_ln_quant(A16, 1, 4, zq.ZQ_MAX_H + 16, A16, A16, 1e-5, A16, A16, None),
     zq.ZQ_ERR_SHAPE),
    (lambda L: L.zq_ln_quant(A16, 2, 4, 64, A16, A16, 1e-5, A16, A16, None), zq.ZQ_ERR_DTYPE),
    (lambda L: L.zq_ln_quant(MIS, 1, 4, 64, A16, A16, 1e-5, A16, A16, None), zq.ZQ_ERR_ALIGN),
    (lambda L: L.zq_ln_quant(A16, 1, 4, 64, A16 + 4, A16, 1e-5, A16, A16, None), zq.ZQ_ERR_ALIGN),
    (lambda L: L.zq_ln_quant(A16, 1, 4, 64, A16, A16, -1.0, A16, A16, None), zq.ZQ_ERR_SHAPE),
    (lambda L: L.zq_act_quant(A16, 1, 4, 64, None, 5, A16, A16, None), zq.ZQ_ERR_DTYPE),
    (lambda L: L.zq_act_quant(A16, 1, 4, 64, MIS, 0, A16, A16, None), zq.ZQ_ERR_ALIGN),
    (lambda L: L.zq_act_quant(A16, 0, 4, 64, None, 0, None, A16, None), zq.ZQ_ERR_NULL),
    (lambda L: L.zq_quantize_weights(None, 64, 64, 16, A16, A16, None), zq.ZQ_ERR_NULL),
    (lambda L: L.zq_quantize_weights(A16, 64, 64, 48, A16, A16, None), zq.ZQ_ERR_SHAPE),
    (lambda L: L.zq_quantize_weights(A16, 64, 40, 16, A16, A16, None), zq.ZQ_ERR_SHAPE),
    (lambda L: L.zq_quantize_weights(A16, 64, 64, 16, MIS, A16, None), zq.ZQ_ERR_ALIGN),
    (lambda L: L.zq_linear_block(A16, 1, 64, 128, A16, A16, 1e-5, A16, A16, 256, 16, None, 0,
                                 zq.ZQ_OUT_BF16, A16, None, None, 0, None), zq.ZQ_ERR_WORKSPACE),
    (lambda L: L.zq_linear_block(A16, 1, 64, 128, A16, None, 1e-5, A16, A16, 256, 16, None, 0,
                                 zq.ZQ_OUT_BF16, A16, None, A16, 1 << 20, None), zq.ZQ_ERR_NULL),
    (lambda L: L.zq_linear_block(A16, 1, 64, 128, A16, A16, 1e-5, A16, A16, 256, 48, None, 0,
                                 zq.ZQ_OUT_BF16, A16, None, A16, 1 << 20, None), zq.ZQ_ERR_SHAPE),
])
def test_row_entry_points_reject_bad_arguments_on_host(call, status):
    assert call(zq.lib()) == status


Z = zq  # short alias for the status and enum names below


@pytest.mark.parametrize("call,status", [
    # SmoothQuant: calibration and fold
    (lambda L: L.zq_smooth_calibrate(None, 1, 64, 768, A16, A16, 1e-5, A16, None), Z.ZQ_ERR_NULL),
    (lambda L: L.zq_smooth_calibrate(A16, 1, 64, 768, A16, A16, 1e-5, None, None), Z.ZQ_ERR_NULL),
    (lambda L: L.zq_smooth_calibrate(A16, 3, 64, 768, A16, A16, 1e-5, A16, None), Z.ZQ_ERR_DTYPE),
    (lambda L: L.zq_smooth_calibrate(A16, 1, 64, 760, A16, A16, 1e-5, A16, None), Z.ZQ_ERR_SHAPE),
    (lambda L: L.zq_smooth_calibrate(A16, 1, 64, 32768 + 16, A16, A16, 1e-5, A16, None), Z.ZQ_ERR_SHAPE),
    (lambda L: L.zq_smooth_calibrate(MIS, 1, 64, 768, A16, A16, 1e-5, A16, None), Z.ZQ_ERR_ALIGN),
    (lambda L: L.zq_smooth_weights(None, 64, 768, A16, 0.5, A16, A16, A16b, A16c, A16c, A16b, None),
     Z.ZQ_ERR_NULL),
    (lambda L: L.zq_smooth_weights(A16, 64, 768, A16, 0.5, A16, A16, A16b, None, A16c, A16b, None),
     Z.ZQ_ERR_NULL),                                   # gamma given, gamma_out missing
    (lambda L: L.zq_smooth_weights(A16, 64, 768, A16, 1.5, A16, A16, A16b, A16c, A16c, A16b, None),
     Z.ZQ_ERR_DTYPE),                                  # alpha outside [0, 1]
    (lambda L: L.zq_smooth_weights(A16, 64, 760, A16, 0.5, A16, A16, A16b, A16c, A16c, A16b, None),
     Z.ZQ_ERR_SHAPE),
    (lambda L: L.zq_smooth_weights(A16, 64, 768, A16, 0.5, A16, A16, MIS, A16c, A16c, A16b, None),
     Z.ZQ_ERR_ALIGN),
    # LLM.int8(): selection, fp16 operands, the linear with the outlier epilogue
    (lambda L: L.zq_llmint8_select(None, 768, 6.0, A16, A16, A16b, A16c, A16, A16, None), Z.ZQ_ERR_NULL),
    (lambda L: L.zq_llmint8_select(A16, 760, 6.0, A16, A16, A16b, A16c, A16, A16, None), Z.ZQ_ERR_SHAPE),
    (lambda L: L.zq_llmint8_select(A16 + 2, 768, 6.0, A16, A16, A16b, A16c, A16, A16, None), Z.ZQ_ERR_ALIGN),
    (lambda L: L.zq_llmint8_outlier_act(A16, 2, 64, 768, A16, A16, 1e-5, A16b, A16c, A16, None),
     Z.ZQ_ERR_DTYPE),
    (lambda L: L.zq_llmint8_outlier_act(A16, 1, 64, 768, A16, A16, 1e-5, A16b, A16c, MIS, None),
     Z.ZQ_ERR_ALIGN),
    (lambda L: L.zq_llmint8_outlier_weights(A16, 256, 768, None, A16c, A16, None), Z.ZQ_ERR_NULL),
    (lambda L: L.zq_llmint8_outlier_weights(A16, 256, 760, A16b, A16c, A16, None), Z.ZQ_ERR_SHAPE),
    (lambda L: L.zq_w8a8_linear_llmint8(A16, A16b, 64, 128, A16c, A16b, 256, 16, None, 0,
                                        Z.ZQ_OUT_I8_REQUANT, A16, A16, A16, None), Z.ZQ_ERR_DTYPE),
    (lambda L: L.zq_w8a8_linear_llmint8(A16, A16b, 64, 128, A16c, A16b, 256, 16, None, 0,
                                        Z.ZQ_OUT_BF16, None, A16, A16, None), Z.ZQ_ERR_NULL),
    (lambda L: L.zq_w8a8_linear_llmint8(A16, A16b, 64, 128, A16c, A16b, 256, 48, None, 0,
                                        Z.ZQ_OUT_BF16, A16, A16, A16, None), Z.ZQ_ERR_SHAPE),
    (lambda L: L.zq_w8a8_linear_llmint8(A16, A16b, 64, 128, A16c, A16b, 256, 16, None, 0,
                                        Z.ZQ_OUT_BF16, MIS, A16, A16, None), Z.ZQ_ERR_ALIGN),
    # the requantizing linear with library-owned scratch
    (lambda L: L.zq_w8a8_linear_requant_noalloc(A16, A16b, 64, 128, A16c, A16b, 256, 16, None, 0, A16, None,
                                                None), Z.ZQ_ERR_NULL),
    (lambda L: L.zq_w8a8_linear_requant_noalloc(A16, A16b, 64, 128, A16c, A16b, 256, 16, None, 2, A16, A16b,
                                                None), Z.ZQ_ERR_DTYPE),
    (lambda L: L.zq_w8a8_linear_requant_noalloc(A16, A16b, 64, 120, A16c, A16b, 256, 16, None, 0, A16, A16b,
                                                None), Z.ZQ_ERR_SHAPE),
    (lambda L: L.zq_w8a8_linear_requant_noalloc(A16, A16b, 64, 128, A16c, A16b, 300000, 16, None, 0, A16,
                                                A16b, None), Z.ZQ_ERR_SCRATCH),   # 77 MB of fp32 rows
    # K-axis weight groups: quantizer and linear
    (lambda L: L.zq_quantize_weights_kgroups(None, 64, 256, 32, A16, A16b, None), Z.ZQ_ERR_NULL),
    (lambda L: L.zq_quantize_weights_kgroups(A16, 64, 250, 25, A16, A16b, None), Z.ZQ_ERR_SHAPE),  # K % 16
    (lambda L: L.zq_quantize_weights_kgroups(A16, 64, 256, 48, A16, A16b, None), Z.ZQ_ERR_SHAPE),  # K % G
    (lambda L: L.zq_quantize_weights_kgroups(A16, 64, 256, 0, A16, A16b, None), Z.ZQ_ERR_SHAPE),
    (lambda L: L.zq_quantize_weights_kgroups(A16, 64, 256, 32, MIS, A16b, None), Z.ZQ_ERR_ALIGN),
    (lambda L: L.zq_quantize_weights_kgroups(A16, 64, 256, 32, A16, A16b + 2, None), Z.ZQ_ERR_ALIGN),
])
def test_extension_entry_points_reject_bad_arguments_on_host(call, status):
    assert call(zq.lib()) == status


def _kg(**kw):
    a = dict(xq=A16, s_tok=A16b, T=64, K=256, Wq=A16c, s_w=A16b, N=256, G=128, bias=None, act=0,
             out=zq.ZQ_OUT_BF16, y=A16, stream=None)
    a.update(kw)
    return zq.lib().zq_w8a8_linear_kgroups(a["xq"], a["s_tok"], a["T"], a["K"], a["Wq"], a["s_w"], a["N"],
                                           a["G"], a["bias"], a["act"], a["out"], a["y"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(xq=None), zq.ZQ_ERR_NULL),
    (dict(s_tok=None), zq.ZQ_ERR_NULL),
    (dict(s_w=None), zq.ZQ_ERR_NULL),
    (dict(y=None), zq.ZQ_ERR_NULL),
    (dict(out=zq.ZQ_OUT_I8_REQUANT), zq.ZQ_ERR_DTYPE),
    (dict(out=zq.ZQ_OUT_I32_RAW), zq.ZQ_ERR_DTYPE),
    (dict(act=2), zq.ZQ_ERR_DTYPE),
    (dict(T=0), zq.ZQ_ERR_SHAPE),
    (dict(G=16), zq.ZQ_ERR_SHAPE),             # narrower than one 32-value k-step
    (dict(G=96), zq.ZQ_ERR_SHAPE),             # K % G
    (dict(K=512, G=512), zq.ZQ_ERR_SHAPE),     # above 256 columns
    (dict(N=250), zq.ZQ_ERR_SHAPE),            # N % 16
    (dict(xq=MIS), zq.ZQ_ERR_ALIGN),
    (dict(Wq=MIS), zq.ZQ_ERR_ALIGN),
    (dict(y=MIS), zq.ZQ_ERR_ALIGN),
    (dict(s_w=A16b + 4), zq.ZQ_ERR_ALIGN),     # scales: 16-byte alignment, as documented
    (dict(bias=A16 + 4), zq.ZQ_ERR_ALIGN),     # bias too (16-byte loads)
    (dict(s_tok=A16b + 2), zq.ZQ_ERR_ALIGN),
])
def test_kgroup_linear_rejects_bad_arguments_on_host(kw, status):
    assert _kg(**kw) == status
