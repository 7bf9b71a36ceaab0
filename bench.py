"""Benchmark of the W8A8 linear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One JSON line on stdout (rank 0).  A step is one pass of the whole inference
path over one batch of seeded synthetic input already resident in HBM; the
default workload is the BERT-base-shaped FFN block:
    x bf16 [4096, 768] -> fused LayerNorm + per-token quant
      -> W1 [3072, 768] INT8 GEMM + dequant + bias + GeLU + per-token requant
      -> W2 [768, 3072] INT8 GEMM + dequant + bias -> bf16 [4096, 768].
Weight group quantization is offline (done once before timing).

Other workloads (--workload): gptj_qkv (LN + 2048x4096 -> 12288, 128-row
weight groups), neox_decode (16 tokens, 6144 -> 24576), tiny, gemm_sweep_<M>,
ln_sweep_<T>_<H>, bert_smooth (SmoothQuant calibration + weight fold),
bert_llmint8 (LLM.int8() decomposition on BERT W1), gptj_qkv_kgroups (the
GPT-J projection with 128-column K-axis weight groups).

Metric: INT8 tera-operations per second of the whole step (2*T*N*K integer
ops per GEMM, summed, over the step time), with the fused LN/token-quant
bandwidth and the per-kernel roofline alongside.

Timing: each step is one CUDA graph of the library's C-ABI calls (the
kernels chained by programmatic dependent launch); every
timed step is preceded by an L2 flush -- a 256 MiB write followed by a read
of the same buffer, so the 126 MB L2 ends up holding only clean lines of the
flush buffer and no write-back of flush data lands inside the timed step --
and is bracketed by CUDA events on the launching stream (the flush is
outside the events).  W >= 3 warm-up steps; K timed steps; barrier + synchronize on both
sides; the maximum over ranks.  Multi-GPU runs are independent replicas
(the path needs no exchange): value = ops of all ranks / max time.  The
per-stage breakdown and the roofline come from a second timed run with one
graph per stage (each stage then pays its own launch latency).

--impl reference times the CPU oracle (the plain C reference of the same
path) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from w8a8_post_quantized_b200 import inputs  # noqa: E402

# Roofline denominators measured on this GPU pool (fallback if the file is absent).
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_INT8_TOPS = 4500.0          # dense INT8 tensor-core peak, spec
SPEC_HBM_GBS = 8000.0
INT8_OVER_BF16 = 2.0             # nominal dense ratio (4.5 / 2.25 PFLOP/s)
L2_FLUSH_BYTES = 256 << 20


class L2Flush:
    """Write then read back a buffer twice the size of L2 (leaves L2 clean)."""

    def __init__(self, torch, device):
        self.buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=device)
        self.sink = torch.empty(1, dtype=torch.int32, device=device)

    def __call__(self):
        self.buf.fill_(1)
        self.sink.copy_(self.buf.max().view(1))


def ridge_ops_per_byte():
    """Ops per byte where the int8 tensor peak meets HBM bandwidth."""
    pk = load_peaks()
    return INT8_OVER_BF16 * pk["bf16_tflops"] * 1e12 / (pk["hbm_gbs"] * 1e9)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


# ------------------------------------------------------------- distributed

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def reduce_max(value: float) -> float:
    """Maximum of a per-rank scalar over all ranks (identity when single-process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    backend = dist.get_backend()
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples (every 200 ms, timestamped) of the GPU this rank
    uses; stats() summarises the samples of one time window."""

    QUERY = ("timestamp,index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)

    def _rows(self):
        from datetime import datetime
        rows = []
        for t_read, ln in list(self.lines):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 11:
                continue
            if self.uuid and self.uuid not in f[2]:
                continue
            try:
                t = datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                t = t_read
            rows.append((t, f))
        return rows

    def stats(self, window=None):
        """Median SM clock under load, max clock and throttle reasons of the
        samples inside `window` (t0, t1) (all samples when None; the nearest
        one when the window holds none)."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = self._rows()
        if window is not None and rows:
            t0, t1 = window
            inside = [r for r in rows if t0 - 0.1 <= r[0] <= t1 + 0.1]
            if not inside:
                mid = 0.5 * (t0 + t1)
                inside = [min(rows, key=lambda r: abs(r[0] - mid))]
            rows = inside
        rows = [f for _, f in rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        num = lambda v: v.replace(".", "").isdigit()
        sm = [float(r[3]) for r in rows if num(r[3])]
        mx = [float(r[4]) for r in rows if num(r[4])]
        reasons = sorted({self.REASONS[i] for r in rows for i in range(4) if r[7 + i] == "Active"})
        loaded = [v for v in sm if mx and v > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------- workloads

class Workload:
    """A workload prepared on the device: stage callables of the public API."""

    def __init__(self, name, zq, torch, device):
        self.name = name
        self.zq, self.torch, self.device = zq, torch, device
        self.stages = []          # (label, fn) run in order; each one stage of the step
        self.ops = 0              # integer ops of the GEMMs per step
        self.tokens = 0
        self.h2d = None           # (pinned host tensor, device tensor) of the step's input
        self.d2h = None           # (device tensor, pinned host tensor) of the step's result
        self.kernel_units = {}    # stage label -> (bound, algorithmic units per launch, unit)
        self.bytes = 0            # algorithmic bytes per step when the metric is bandwidth
        self.metric = None
        self.config = {}

    def dev(self, a):
        if isinstance(a, self.torch.Tensor):      # drawn on the device already
            return a
        return self.torch.from_numpy(np.ascontiguousarray(a)).to(self.device)

    def dev_act(self, a):
        if isinstance(a, self.torch.Tensor):
            return a
        if a.bf16 is not None:
            return self.torch.from_numpy(a.bf16.view(np.int16)).to(self.device).view(self.torch.bfloat16)
        return self.dev(a.f32)


def build_smooth_workload(W, zq, torch, device):
    """SmoothQuant offline steps on the BERT-base FFN's first linear: the
    calibration pass over the LayerNorm output of the 4096-token batch and
    the factor + fold of W1 [3072, 768] (and gamma, beta).  HBM-bound."""
    w = inputs.bert_ffn()
    lin = w.layers[0]
    x = W.dev_act(w.x)
    T, H = x.shape
    g, b = W.dev(w.gamma), W.dev(w.beta)
    W1 = W.dev(lin.W)
    N = W1.shape[0]
    amax = torch.zeros(H, dtype=torch.float32, device=device)
    W1o, go, bo = torch.empty_like(W1), torch.empty_like(g), torch.empty_like(b)
    sf = torch.empty(H, dtype=torch.float32, device=device)
    # the calibration is a running max: repeating it on the same batch is idempotent
    W.stages.append(("smooth_calibrate", lambda: zq.zq_smooth_calibrate(x, g, b, w.eps, amax=amax)))
    W.stages.append(("smooth_weights", lambda: zq.zq_smooth_weights(W1, amax, 0.5, g, b, W_out=W1o,
                                                                     gamma_out=go, beta_out=bo, s=sf)))
    xbytes = x.numel() * x.element_size()
    # algorithmic bytes: x, gamma, beta read once, amax read and written;
    # W read once and W' written once, plus the per-channel vectors
    W.kernel_units["smooth_calibrate"] = ("hbm", xbytes + 8 * H + 8 * H, "bytes")
    W.kernel_units["smooth_weights"] = ("hbm", 8 * N * H + 6 * 4 * H, "bytes")
    W.bytes = sum(v[1] for v in W.kernel_units.values())
    W.metric = "SmoothQuant calibration + weight fold GB/s (algorithmic bytes)"
    W.tokens = T
    W.h2d_src = x
    W.out = sf
    W.config = {"workload": "bert_ffn W1 SmoothQuant (calibrate LN output 4096x768 bf16, fold W1 3072x768)",
                "tokens": T, "hidden": H, "x_dtype": w.x.dtype, "alpha": 0.5}
    return W


def build_llmint8_workload(W, zq, torch, device):
    """LLM.int8() decomposition on the BERT-base FFN's first linear, per batch:
    column absmax of the LayerNorm output, outlier selection (alpha = 6) with
    masked LayerNorm parameters, LN + token quant of the other columns, the
    fp16 outlier operands, and the W8A8 GEMM whose epilogue adds the outlier
    product (+ bias + GeLU, bf16 out)."""
    w = inputs.bert_ffn()
    lin = w.layers[0]
    x = W.dev_act(w.x)
    T, H = x.shape
    g, b = W.dev(w.gamma), W.dev(w.beta)
    W1 = W.dev(lin.W)
    N = W1.shape[0]
    G = lin.group_rows
    Wq, sg = zq.zq_quantize_weights(W1, G)
    bias = W.dev(lin.bias)
    amax = torch.zeros(H, dtype=torch.float32, device=device)
    idx = torch.empty(zq.ZQ_LLMINT8_MAX_OUTLIERS, dtype=torch.int32, device=device)
    count = torch.empty(1, dtype=torch.int32, device=device)
    gm, bm = torch.empty_like(g), torch.empty_like(b)
    q = torch.empty((T, H), dtype=torch.int8, device=device)
    st = torch.empty(T, dtype=torch.float32, device=device)
    xo = torch.empty((T, zq.ZQ_LLMINT8_MAX_OUTLIERS), dtype=torch.float16, device=device)
    wo = torch.empty((N, zq.ZQ_LLMINT8_MAX_OUTLIERS), dtype=torch.float16, device=device)
    y = torch.empty((T, N), dtype=torch.bfloat16, device=device)
    P = zq.lib()

    def detect():
        # the per-batch column absmax is a running max: restart it from zero
        amax.zero_()
        zq.zq_smooth_calibrate(x, g, b, w.eps, amax=amax)
        zq._check(P.zq_llmint8_select(zq._p(amax), H, 6.0, zq._p(g), zq._p(b), zq._p(idx), zq._p(count),
                                      zq._p(gm), zq._p(bm), zq._s(None)), "zq_llmint8_select")

    def operands():
        zq.zq_ln_quant(x, gm, bm, w.eps, q=q, s_tok=st)
        zq._check(P.zq_llmint8_outlier_act(zq._p(x), zq._dtype_code(x), T, H, zq._p(g), zq._p(b), float(w.eps),
                                           zq._p(idx), zq._p(count), zq._p(xo), zq._s(None)),
                  "zq_llmint8_outlier_act")
        zq._check(P.zq_llmint8_outlier_weights(zq._p(W1), N, H, zq._p(idx), zq._p(count), zq._p(wo), zq._s(None)),
                  "zq_llmint8_outlier_weights")

    W.stages.append(("detect", detect))
    W.stages.append(("operands", operands))
    W.stages.append(("linear1", lambda: zq.zq_w8a8_linear_llmint8(q, st, Wq, sg, G, xo, wo, bias=bias, act=1,
                                                                   out_kind=zq.ZQ_OUT_BF16, y=y)))
    xbytes = x.numel() * x.element_size()
    W.kernel_units["detect"] = ("hbm", xbytes + 8 * H + 4 * H, "bytes")
    W.kernel_units["operands"] = ("hbm", 2 * xbytes + T * H + 4 * T + 16 * T + 16 * N, "bytes")
    ops = 2 * T * N * H + 2 * T * N * zq.ZQ_LLMINT8_MAX_OUTLIERS
    W.kernel_units["linear1"] = ("tensor", ops, "ops")
    W.ops = 2 * T * N * H
    W.tokens = T
    W.h2d_src = x
    W.out = y
    W.config = {"workload": "bert_ffn W1 with LLM.int8() decomposition (alpha 6, up to 8 fp16 columns)",
                "tokens": T, "hidden": H, "x_dtype": w.x.dtype, "epilogue": "fp16 outliers + bias + gelu",
                "out_dtype": "bf16"}
    return W


KGROUP_COLS = 128


def build_kgroup_workload(W, zq, torch, device):
    """The GPT-J-6B QKV projection (2048 tokens, 4096 -> 12288, bf16 out) with
    K-axis weight groups: LN + token quant, then the INT8 GEMM whose epilogue
    scales every 128-column group's partial product as it completes."""
    w = inputs.gptj_qkv()
    lin = w.layers[0]
    x = W.dev_act(w.x)
    T, K = x.shape
    N = lin.W.shape[0]
    G = KGROUP_COLS
    g, b = W.dev(w.gamma), W.dev(w.beta)
    q1 = torch.empty((T, K), dtype=torch.int8, device=device)
    st1 = torch.empty(T, dtype=torch.float32, device=device)
    Wq, sw = zq.zq_quantize_weights_kgroups(W.dev(lin.W), G)
    bias = W.dev(lin.bias)
    y = torch.empty((T, N), dtype=torch.bfloat16, device=device)
    torch.cuda.synchronize()
    W.stages.append(("ln_quant", lambda: zq.zq_ln_quant(x, g, b, w.eps, q=q1, s_tok=st1)))
    W.stages.append(("linear1", lambda: zq.zq_w8a8_linear_kgroups(q1, st1, Wq, sw, G, bias=bias,
                                                                   out_kind=zq.ZQ_OUT_BF16, y=y)))
    xbytes = x.numel() * x.element_size()
    W.kernel_units["ln_quant"] = ("hbm", xbytes + T * K + 4 * T + 8 * K, "bytes")
    ops = 2 * T * N * K
    W.kernel_units["linear1"] = ("tensor", ops, "ops")
    W.ops = ops
    W.tokens = T
    W.h2d_src = x
    W.out = y
    W.config = {"workload": f"gptj_6b_qkv_{T}x{K}x{N}_kgroups{G}", "tokens": T, "hidden": K,
                "x_dtype": w.x.dtype, "layers": [[N, K, G]], "weight_groups": f"{G} input columns per scale",
                "epilogue": "per-group scale, bias", "out_dtype": "bf16"}
    return W


def _device_inputs(name, device):
    """The workload drawn on the GPU (same shapes and distributions as the
    numpy recipe; used for the large sub-records of the default run)."""
    from w8a8_post_quantized_b200 import inputs_device as idev
    if name == "gptj_qkv":
        return idev.gptj_qkv(device)
    if name == "gptj_ffn":
        return idev.gptj_ffn(device)
    if name == "neox_decode":
        return idev.neox_decode(device)
    if name.startswith("gemm_sweep_"):
        M = int(name.split("_")[-1])
        return idev.gemm_sweep_point(device, M, inputs.GEMM_SWEEP_M.index(M))
    if name.startswith("ln_sweep_"):
        T, H = (int(v) for v in name.split("_")[-2:])
        idx = inputs.LN_SWEEP_T.index(T) * len(inputs.LN_SWEEP_H) + inputs.LN_SWEEP_H.index(H)
        return idev.ln_sweep_point(device, T, H, idx)
    raise SystemExit(f"no device generator for {name}")


def _x_dtype(x):
    if hasattr(x, "dtype") and isinstance(x.dtype, str):
        return x.dtype
    return "bf16" if str(x.dtype).endswith("bfloat16") else "f32"


def build_workload(name, zq, torch, device, source="host"):
    W = Workload(name, zq, torch, device)
    if source == "device":
        return build_linear_workload(W, _device_inputs(name, device), zq, torch, device)
    if name == "gptj_qkv_kgroups":
        return build_kgroup_workload(W, zq, torch, device)
    if name == "bert_smooth":
        return build_smooth_workload(W, zq, torch, device)
    if name == "bert_llmint8":
        return build_llmint8_workload(W, zq, torch, device)
    if name in ("bert_ffn", "gptj_qkv", "tiny"):
        w = {"bert_ffn": inputs.bert_ffn, "gptj_qkv": inputs.gptj_qkv, "tiny": inputs.tiny}[name]()
    elif name == "neox_decode":
        w = inputs.neox_decode()
    elif name.startswith("gemm_sweep_"):
        M = int(name.split("_")[-1])
        w = inputs.gemm_sweep_point(M, inputs.GEMM_SWEEP_M.index(M))
    elif name.startswith("ln_sweep_"):
        T, H = (int(v) for v in name.split("_")[-2:])
        idx = inputs.LN_SWEEP_T.index(T) * len(inputs.LN_SWEEP_H) + inputs.LN_SWEEP_H.index(H)
        w = inputs.ln_sweep_point(T, H, idx)
    elif name == "gptj_ffn":
        return build_linear_workload(W, _device_inputs(name, device), zq, torch, device)
    else:
        raise SystemExit(f"unknown workload {name}")
    return build_linear_workload(W, w, zq, torch, device)


def build_linear_workload(W, w, zq, torch, device):
    """Quantizer (LN + quant, or plain token quant) followed by the workload's
    linears; every linear but the last requantizes its output per token."""
    x = W.dev_act(w.x)
    T, K = x.shape
    W.tokens = T
    xbytes = x.numel() * x.element_size()
    W.config = {"workload": w.name, "tokens": T, "hidden": K, "x_dtype": _x_dtype(w.x)}
    q1 = torch.empty((T, K), dtype=torch.int8, device=device)
    st1 = torch.empty(T, dtype=torch.float32, device=device)
    if w.gamma is not None:
        g, b = W.dev(w.gamma), W.dev(w.beta)
        W.stages.append(("ln_quant", lambda: zq.zq_ln_quant(x, g, b, w.eps, q=q1, s_tok=st1)))
        label_q = "ln_quant"
    else:
        W.stages.append(("act_quant", lambda: zq.zq_act_quant(x, q=q1, s_tok=st1)))
        label_q = "act_quant"
    # algorithmic bytes of the quantizer: read x, write codes and scales (+ gamma, beta)
    W.kernel_units[label_q] = ("hbm", xbytes + T * K + 4 * T + (8 * K if w.gamma is not None else 0),
                               "bytes")
    W.h2d_src = x
    if not w.layers:          # LN sweep point: the quantizer alone
        W.out = q1
        W.config.update(layers=[])
        return W
    layers = []
    for lin in w.layers:
        Wq, sg = zq.zq_quantize_weights(W.dev(lin.W), lin.group_rows)
        layers.append((Wq, sg, W.dev(lin.bias), lin.group_rows))
        lin.W = None          # the fp32 weights are not needed once quantized
    torch.cuda.synchronize()
    a_q, a_s = q1, st1
    for i, (Wq, sg, b, G) in enumerate(layers):
        N = Wq.shape[0]
        last = i == len(layers) - 1
        act = w.act if i == 0 else 0
        if last:
            out_kind = {"bf16": zq.ZQ_OUT_BF16, "f32": zq.ZQ_OUT_F32}[w.out]
            y = torch.empty((T, N), dtype=torch.bfloat16 if w.out == "bf16" else torch.float32,
                            device=device)
            s_out = None
        else:
            out_kind = zq.ZQ_OUT_I8_REQUANT
            y = torch.empty((T, N), dtype=torch.int8, device=device)
            s_out = torch.empty(T, dtype=torch.float32, device=device)
        # allocated once, outside the timed region (a few-token layer's
        # partial sums, a requantizing layer's row statistics)
        ws_bytes = zq.zq_w8a8_linear_workspace(T, Wq.shape[1], N, out_kind)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=device) if ws_bytes else None

        def fn(a_q=a_q, a_s=a_s, Wq=Wq, sg=sg, b=b, G=G, act=act, out_kind=out_kind, y=y,
               s_out=s_out, ws=ws):
            zq.zq_w8a8_linear(a_q, a_s, Wq, sg, G, bias=b, act=act, out_kind=out_kind, y=y,
                              s_tok_out=s_out, workspace=ws)
        label = f"linear{i + 1}"
        W.stages.append((label, fn))
        Kd = Wq.shape[1]
        ops = 2 * T * N * Kd
        W.ops += ops
        # algorithmic bytes: activations and weights in once, outputs out once
        out_b = T * N * (1 if out_kind == zq.ZQ_OUT_I8_REQUANT else y.element_size()) + \
            (4 * T if out_kind == zq.ZQ_OUT_I8_REQUANT else 0)
        lin_bytes = T * Kd + 4 * T + N * Kd + 4 * (N // G) + (4 * N if b is not None else 0) + out_b
        # the roofline that binds: HBM when the ops per byte fall below the
        # ridge point (int8 peak / HBM bandwidth), the tensor cores otherwise
        if ops / lin_bytes < ridge_ops_per_byte():
            W.kernel_units[label] = ("hbm", lin_bytes, "bytes")
        else:
            W.kernel_units[label] = ("tensor", ops, "ops")
        a_q, a_s = y, s_out
        W.out = y
    W.config.update(layers=[list(l[0].shape) + [l[3]] for l in layers],
                    epilogue=("gelu+requant" if len(layers) > 1 else ("gelu" if w.act else "bias")),
                    out_dtype=w.out)
    return W


# ------------------------------------------------------------------ timing

def time_device(W, steps, warmup, torch, min_window_s=0.0):
    """Flush L2 before each step; CUDA events on the launching stream.

    The step time comes from one CUDA graph holding the whole step (its
    kernels chained by programmatic dependent launch, as a serving loop would
    replay them), each replay preceded by an L2 flush outside the events.

    The per-stage kernel times come from graphs of [flush; stage] and of
    [flush] alone, each replayed `steps` times between two events: the
    stage's time is the difference divided by `steps`.  Both graphs pay the
    same launch cost, so it cancels, and every stage launch starts on a cold
    L2, as in the step.  With min_window_s > 0 the number of timed steps
    grows until the step timing spans at least that long (so clock samples
    fall inside it).  Returns (per-step ms list, {stage: ms}, steps timed)."""
    stream = torch.cuda.current_stream()
    flush = L2Flush(torch, W.device)
    for _, fn in W.stages:       # eager warm-up (sets kernel attributes, loads modules)
        fn()
    torch.cuda.synchronize()
    cap = torch.cuda.Stream()
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        flush_g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(flush_g, stream=cap):
            flush()
        graphs = []
        for label, fn in W.stages:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                flush()
                fn()
            graphs.append((label, g))
        whole = torch.cuda.CUDAGraph()
        with torch.cuda.graph(whole, stream=cap):
            for _, fn in W.stages:
                fn()
    stream.wait_stream(cap)
    torch.cuda.synchronize()

    def run_step(k):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(k)]
        for s in range(k):
            flush()
            evs[s][0].record(stream)
            whole.replay()
            evs[s][1].record(stream)
        return evs

    def replay_ms(g, k):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(k):
            g.replay()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b)

    evs = run_step(warmup)
    torch.cuda.synchronize()
    if min_window_s > 0:
        est = statistics.median(a.elapsed_time(b) for a, b in evs) + replay_ms(flush_g, 3) / 3
        steps = max(steps, min(4000, int(math.ceil(min_window_s * 1e3 / max(est, 1e-3)))))
    barrier()
    torch.cuda.synchronize()
    evs = run_step(steps)
    torch.cuda.synchronize()
    barrier()
    per_step = [a.elapsed_time(b) for a, b in evs]
    k = max(steps, 20)
    for _, g in graphs:
        replay_ms(g, 2)
    stage_ms = {}
    for label, g in graphs:
        diffs = [(replay_ms(g, k) - replay_ms(flush_g, k)) / k for _ in range(3)]
        stage_ms[label] = max(statistics.median(diffs), 1e-4)
    del graphs, whole, flush_g
    return per_step, stage_ms, steps


def time_e2e(W, steps, warmup, torch):
    """Same step through the public API with host buffers: pinned host input
    -> device, the stage calls, result -> pinned host, all inside the events.
    The step (both copies and the C-ABI calls) is captured once as a CUDA
    graph and replayed, so host-side call overhead stays out of the timed
    region as in a serving loop; the L2 is flushed before every timed step,
    outside the events.  (Row slices of the batch on separate copy-in,
    compute and copy-out streams, so that copies overlap the calls, measured
    slower here: 0.46-0.55 ms against 0.43 ms for the BERT block.)
    Returns (ms per step, H2D bytes, D2H bytes, mode)."""
    stream = torch.cuda.current_stream()
    src = W.h2d_src
    host_in = torch.empty(src.shape, dtype=src.dtype, pin_memory=True)
    host_in.copy_(src.cpu())
    out = W.out
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    flush = L2Flush(torch, W.device)

    def step():
        src.copy_(host_in, non_blocking=True)
        for _, fn in W.stages:
            fn()
        host_out.copy_(out, non_blocking=True)

    for _ in range(warmup):
        flush()
        step()
    torch.cuda.synchronize()
    mode = "graph"
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        torch.cuda.synchronize()
        run = g.replay
    except Exception:  # capture refused: time the eager calls instead
        torch.cuda.synchronize()
        mode, run = "eager", step
    for _ in range(warmup):
        flush()
        run()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        run()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    h2d = host_in.numel() * host_in.element_size()
    d2h = host_out.numel() * host_out.element_size()
    return statistics.mean(times), h2d, d2h, mode


def count_launches(W, zq, torch):
    """Kernels of this library launched per step, in total and per stage."""
    per_stage = {}
    for label, fn in W.stages:
        before = zq.zq_launch_count()
        fn()
        per_stage[label] = zq.zq_launch_count() - before
    torch.cuda.synchronize()
    return sum(per_stage.values()), per_stage


# The sources of the hot-path kernels the ncu records describe (the
# quantizers, both GEMMs, their shared helpers and their launch code).
PROFILED_SOURCES = ("zq_internal.cuh", "zq_api.cu", "zq_rowquant.cu", "zq_quant.cu", "zq_gemm.cu",
                    "zq_gemm_creq.cu", "zq_gemm_greq.cu", "zq_gemm_sk.cu")
# ... and of the K-axis group linear (its kernel, helpers, tensor-map code)
KGROUP_SOURCES = ("zq_internal.cuh", "zq_kgroup.cu", "zq_gemm.cu")


def kernel_source_hash(sources=PROFILED_SOURCES):
    """Hash of the hot-path kernel sources: ncu counters recorded for another
    version of those kernels are not reported."""
    import hashlib
    h = hashlib.sha256()
    for f in sorted(os.path.join(ROOT, "w8a8_post_quantized_b200", "csrc", n) for n in sources):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, stage):
    """DRAM bytes per launch of the stage's kernel from a committed ncu capture
    (profiles/dram_traffic.json), if it was taken on the current version of
    the source files the record lists."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{workload}:{stage}")
    # the record names the source files its hash covers
    if not e or e.get("source_hash") != kernel_source_hash(tuple(e.get("sources", PROFILED_SOURCES))):
        return None
    return e.get("dram_bytes")


# ---------------------------------------------------------- CPU baseline

def oracle_sample(name, budget_s=12.0, max_rows=None):
    """Time the CPU oracle on a bounded row sample of the workload.  Returns
    (ops done, seconds, rows, total rows).  The oracle is single-threaded."""
    import oracle
    if name == "bert_ffn":
        w = inputs.bert_ffn()
    elif name == "gptj_qkv":
        w = inputs.gptj_qkv()
    elif name == "neox_decode":
        w = inputs.neox_decode()
    elif name == "tiny":
        w = inputs.tiny()
    elif name.startswith("gemm_sweep_"):
        M = int(name.split("_")[-1])
        w = inputs.gemm_sweep_point(M, inputs.GEMM_SWEEP_M.index(M))
    elif name == "bert_smooth":
        return oracle_smooth_sample(budget_s, max_rows)
    elif name == "bert_llmint8":
        return oracle_llmint8_sample(budget_s, max_rows)
    elif name == "gptj_qkv_kgroups":
        return oracle_kgroup_sample(budget_s, max_rows)
    else:
        raise SystemExit(f"no oracle baseline for {name}")
    qlayers = [(*oracle.quantize_weights(l.W, l.group_rows), l.bias, l.group_rows) for l in w.layers]
    T = w.x.f32.shape[0]
    rows_done, ops, t_total = 0, 0, 0.0
    chunk = 8 if T >= 8 else T
    limit = max_rows if max_rows is not None else T
    while rows_done < limit and t_total < budget_s:
        r0 = rows_done % T
        x = w.x.f32[r0:r0 + chunk]
        t0 = time.perf_counter()
        if w.gamma is not None:
            q, s = oracle.ln_quant(x, w.gamma, w.beta, w.eps)
        else:
            q, s = oracle.quantize_rows(x)
        for i, (Wq, sg, b, G) in enumerate(qlayers):
            act = w.act if i == 0 else 0
            if i < len(qlayers) - 1:
                q, s = oracle.linear_requant(q, s, Wq, sg, G, b, act)
            else:
                oracle.linear(q, s, Wq, sg, G, b, act)
            ops += 2 * x.shape[0] * Wq.shape[0] * Wq.shape[1]
        t_total += time.perf_counter() - t0
        rows_done += x.shape[0]
    return ops, t_total, rows_done, T


def oracle_smooth_sample(budget_s=12.0, max_rows=None):
    """The oracle's SmoothQuant steps on a bounded sample: the calibration of
    a row sample of the BERT batch, then the factors and fold of all of W1.
    Returns (algorithmic bytes done, seconds, rows, total rows)."""
    import oracle
    w = inputs.bert_ffn()
    lin = w.layers[0]
    T, H = w.x.f32.shape
    N = lin.W.shape[0]
    e = 2 if w.x.dtype == "bf16" else 4
    rows_done, nbytes, t_total = 0, 0, 0.0
    limit = max_rows if max_rows is not None else T
    amax = None
    while rows_done < limit and t_total < budget_s * 0.5:
        x = w.x.f32[rows_done % T:rows_done % T + 8]
        t0 = time.perf_counter()
        amax = oracle.channel_absmax(oracle.layernorm(x, w.gamma, w.beta, w.eps), amax)
        t_total += time.perf_counter() - t0
        rows_done += x.shape[0]
        nbytes += x.shape[0] * H * e
    t0 = time.perf_counter()
    s = oracle.smooth_factors(amax, oracle.weight_col_absmax(lin.W), 0.5)
    oracle.smooth_fold(lin.W, s, w.gamma, w.beta)
    t_total += time.perf_counter() - t0
    nbytes += 8 * N * H + 16 * H
    return nbytes, t_total, rows_done, T


def oracle_llmint8_sample(budget_s=12.0, max_rows=None):
    """The oracle's LLM.int8() layer (BERT W1, GeLU) on row chunks of the BERT
    batch (outliers detected on each chunk).  Returns (ops, seconds, rows, T)."""
    import oracle
    w = inputs.bert_ffn()
    lin = w.layers[0]
    Wq, sg = oracle.quantize_weights(lin.W, lin.group_rows)
    T, H = w.x.f32.shape
    N = lin.W.shape[0]
    rows_done, ops, t_total = 0, 0, 0.0
    limit = max_rows if max_rows is not None else T
    while rows_done < limit and t_total < budget_s:
        x = w.x.f32[rows_done % T:rows_done % T + 8]
        t0 = time.perf_counter()
        oracle.int8_decomposed_ln_linear(x, w.gamma, w.beta, w.eps, lin.W, Wq, sg, lin.group_rows, lin.bias,
                                         oracle.ACT_GELU)
        t_total += time.perf_counter() - t0
        rows_done += x.shape[0]
        ops += 2 * x.shape[0] * N * H
    return ops, t_total, rows_done, T


def oracle_kgroup_sample(budget_s=12.0, max_rows=None):
    """The oracle's LN + token quant + K-group linear (GPT-J QKV, 128-column
    groups) on row chunks.  Returns (ops, seconds, rows, T)."""
    import oracle
    w = inputs.gptj_qkv()
    lin = w.layers[0]
    Wq, sw = oracle.quantize_weights_kgroups(lin.W, KGROUP_COLS)
    T, K = w.x.f32.shape
    N = lin.W.shape[0]
    rows_done, ops, t_total = 0, 0, 0.0
    limit = max_rows if max_rows is not None else T
    while rows_done < limit and t_total < budget_s:
        x = w.x.f32[rows_done % T:rows_done % T + 4]
        t0 = time.perf_counter()
        oracle.ln_linear_kgroups(x, w.gamma, w.beta, w.eps, Wq, sw, KGROUP_COLS, lin.bias)
        t_total += time.perf_counter() - t0
        rows_done += x.shape[0]
        ops += 2 * x.shape[0] * N * K
    return ops, t_total, rows_done, T


# -------------------------------------------------------------------- main

# Sub-records of the default run: the other workloads, each timed on its own
# after the headline (inputs drawn on the device).  GEMM sweep M = 16 / 256
# are HBM-bound (weight stream), M = 4096 / 16384 tensor-bound; the LN sweep
# points are those of at least 32 MB of input.
SUBRECORDS = ("gptj_qkv", "gptj_ffn", "neox_decode", "gemm_sweep_16", "gemm_sweep_256", "gemm_sweep_4096",
              "gemm_sweep_16384", "ln_sweep_16384_1024", "ln_sweep_16384_4096", "ln_sweep_16384_12288",
              "ln_sweep_65536_1024", "ln_sweep_65536_4096", "ln_sweep_65536_12288")


def stage_roofline(W, label, ms, peaks, workload):
    """Achieved rate of one stage's kernel(s) against the roofline that binds it."""
    bound, units, _ = W.kernel_units[label]
    int8_peak = peaks["bf16_tflops"] * INT8_OVER_BF16
    if bound == "tensor":
        achieved = units / (ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(int8_peak, 1), "unit": "TOPS",
                "frac": round(achieved / int8_peak, 4),
                "peak_source": f"{peaks['source']} bf16 burst x {INT8_OVER_BF16:g} (nominal int8/bf16)",
                "frac_vs_spec": round(achieved / SPEC_INT8_TOPS, 4),
                "traffic": recorded_traffic(workload, label), "kernel_ms": round(ms, 5)}
    achieved = units / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(achieved / peaks["hbm_gbs"], 4), "peak_source": f"{peaks['source']} copy bandwidth",
            "frac_vs_spec": round(achieved / SPEC_HBM_GBS, 4),
            "traffic": recorded_traffic(workload, label), "kernel_ms": round(ms, 5)}


def step_value(W, ms_per_step, world=1):
    """(metric, unit, value) of the whole step: INT8 TOPS when the step has
    GEMMs, else GB/s of algorithmic bytes."""
    if W.ops:
        return ("W8A8 linear INT8 TOPS (whole step, incl. fused LN/token-quant)", "TOPS",
                world * W.ops / (ms_per_step * 1e-3) / 1e12)
    qb = sum(v[1] for v in W.kernel_units.values() if v[0] == "hbm")
    return (W.metric or "fused LN/token-quant GB/s", "GB/s", world * (W.bytes or qb) / (ms_per_step * 1e-3) / 1e9)


def dominant_stage(stage_ms, stage_launches):
    """The longest stage.  Some stages launch a one-block kernel that clears
    flags or counters before their main kernel (the few-token even split, the
    grid-exchange requant); their time then covers both launches, which
    understates the main kernel's rate slightly rather than overstating it."""
    return max(stage_ms, key=lambda k: stage_ms[k])


def measure_subrecord(name, zq, torch, device, steps, warmup, peaks, clocks):
    W = build_workload(name, zq, torch, device, source="device")
    launches, stage_launches = count_launches(W, zq, torch)
    t0 = time.time()
    per_step, stage_ms, n = time_device(W, steps, warmup, torch, min_window_s=0.3)
    t1 = time.time()
    zq.zq_device_status()
    ms = statistics.mean(per_step)
    metric, unit, value = step_value(W, ms)
    dom = dominant_stage(stage_ms, stage_launches)
    rec = {"value": round(value, 2), "unit": unit, "ms_per_step": round(ms, 5), "steps": n,
           "tokens_per_s": round(W.tokens / (ms * 1e-3), 1),
           "config": dict(W.config, inputs="drawn on the device (torch CUDA generator), numpy recipe's distributions"),
           "stages_ms": {k: round(v, 5) for k, v in stage_ms.items()},
           "stage_roofline": {k: stage_roofline(W, k, v, peaks, name) for k, v in stage_ms.items()},
           "dominant": dom, "gpu_launches": launches * n, "clocks": clocks.stats((t0, t1))}
    rec["roofline"] = dict(rec["stage_roofline"][dom], kernel=dom, launches_in_stage=stage_launches.get(dom))
    del W
    torch.cuda.empty_cache()
    return rec


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="bert_ffn")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-subrecords", action="store_true",
                    help="time only the selected workload (default run: also the other workloads)")
    ap.add_argument("--subrecords", default=None, help="comma-separated sub-record workloads to time")
    ap.add_argument("--inputs", default="host", choices=["host", "device"],
                    help="draw the selected workload's inputs with numpy (host) or on the GPU (device)")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank, world, local_rank = dist_env()

    if a.impl == "reference":
        return main_reference(a, rank, world)

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    from w8a8_post_quantized_b200 import zq
    zq.lib()

    W = build_workload(a.workload, zq, torch, device, source=a.inputs)
    launches_per_step, stage_launches = count_launches(W, zq, torch)
    zq.zq_device_status()

    props = torch.cuda.get_device_properties(device)
    clocks = ClockSampler(str(getattr(props, "uuid", "")) or None)
    clocks.start()
    t0 = time.time()
    per_step, stage_ms, _ = time_device(W, a.steps, a.warmup, torch)
    t1 = time.time()
    zq.zq_device_status()
    local_ms = sum(per_step)
    max_ms = reduce_max(local_ms)
    ms_per_step = max_ms / a.steps

    e2e_ms, h2d, d2h, e2e_mode = time_e2e(W, max(3, min(a.steps, 20)), 3, torch)
    e2e_ms = reduce_max(e2e_ms)
    zq.zq_device_status()

    peaks = load_peaks()
    dom = dominant_stage(stage_ms, stage_launches)
    roof = dict(stage_roofline(W, dom, stage_ms[dom], peaks, a.workload),
                kernel=f"w8a8 linear ({dom})" if dom.startswith("linear") else dom,
                launches_in_stage=stage_launches.get(dom))
    qlabel = "ln_quant" if "ln_quant" in stage_ms else ("act_quant" if "act_quant" in stage_ms else None)
    qb = W.kernel_units[qlabel][1] if qlabel else 0
    q_gbs = qb / (stage_ms[qlabel] * 1e-3) / 1e9 if qlabel else None

    metric, unit, value = step_value(W, ms_per_step, world)
    e2e_value = value * ms_per_step / e2e_ms

    out = {
        "metric": metric, "value": round(value, 2), "unit": unit, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8" if W.ops or W.metric is None else "f32",
        "data": "synthetic (seeded; layer shapes only, random weights)",
        "config": dict(W.config, parallelism=f"replicas x{world}",
                       l2="flushed before every timed step (256 MiB write + read-back)",
                       timing="one CUDA graph per step (kernels chained by programmatic dependent launch), "
                              "CUDA events on the launching stream; per-stage kernel times from graphs of "
                              "[flush; stage] minus graphs of [flush], replayed back to back"),
        "tokens_per_s": round(world * W.tokens / (ms_per_step * 1e-3), 1),
        "stages_ms": {k: round(v, 5) for k, v in stage_ms.items()},
        "stage_roofline": {k: stage_roofline(W, k, v, peaks, a.workload) for k, v in stage_ms.items()},
        "ln_quant_gbs": round(q_gbs, 1) if q_gbs else None,
        "ln_quant_frac_hbm": round(q_gbs / peaks["hbm_gbs"], 4) if q_gbs else None,
        "roofline": roof,
        "e2e": {"value": round(e2e_value, 3), "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "timing": f"{e2e_mode}: pinned host in -> C-ABI calls -> pinned host out per step, "
                          "L2 flushed before each step outside the events"},
        "gpu_launches": launches_per_step * a.steps,
        "launches_per_stage": stage_launches,
        "clocks": clocks.stats((t0, t1)),
    }
    has_ops = bool(W.ops)
    del W
    torch.cuda.empty_cache()
    # the other workloads, one GPU only (replica runs time the headline alone)
    names = SUBRECORDS if a.subrecords is None else tuple(n for n in a.subrecords.split(",") if n)
    if world == 1 and a.workload == "bert_ffn" and not a.no_subrecords and names:
        subs = {}
        for name in names:
            subs[name] = measure_subrecord(name, zq, torch, device, max(10, min(a.steps, 20)), a.warmup, peaks,
                                           clocks)
        out["subrecords"] = subs
        out["clocks_all"] = clocks.stats()
    clocks.stop()
    if rank == 0 and world == 1 and not a.no_cpu_baseline and has_ops:
        ops, secs, rows, T = oracle_sample(a.workload, budget_s=a.cpu_budget)
        out["cpu_baseline"] = {"value": round(ops / secs / 1e12, 8), "unit": unit, "cores": 1,
                               "kind": "oracle",
                               "sample": f"{rows} of {T} token rows of {out['config']['workload']}, "
                                         f"plain C oracle, single thread, {secs:.1f} s"}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main_reference(a, rank, world):
    """The CPU oracle as the reference arm: rank 0 only, bounded samples."""
    if rank != 0:
        return 0
    ops_tot, secs_tot, rows_tot = 0, 0.0, 0
    per_step_budget = max(0.5, min(8.0, 120.0 / max(1, a.steps + a.warmup)))
    T = 0
    for i in range(a.warmup + a.steps):
        ops, secs, rows, T = oracle_sample(a.workload, budget_s=per_step_budget, max_rows=64)
        if i >= a.warmup:
            ops_tot += ops
            secs_tot += secs
            rows_tot += rows
    if a.workload == "bert_smooth":
        value = ops_tot / secs_tot / 1e9
        metric, unit = "SmoothQuant calibration + weight fold GB/s (algorithmic bytes)", "GB/s"
    else:
        value = ops_tot / secs_tot / 1e12
        metric, unit = "W8A8 linear INT8 TOPS (whole step, incl. fused LN/token-quant)", "TOPS"
    out = {"impl": "reference", "metric": metric, "value": round(value, 8), "unit": unit,
           "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
           "ms_per_step": round(1e3 * secs_tot / a.steps, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f32" if a.workload == "bert_smooth" else "int8",
           "data": "synthetic",
           "config": {"workload": a.workload, "sample_rows_per_step": rows_tot // max(1, a.steps),
                      "total_rows": T},
           "cpu_baseline": {"value": round(value, 8), "unit": unit, "cores": 1, "kind": "oracle",
                            "sample": f"{rows_tot // max(1, a.steps)} token rows per step of {T}"},
           "e2e": {"value": round(value, 8), "unit": unit, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
