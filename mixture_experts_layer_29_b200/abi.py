"""Python binding of the C ABI in include/moe.h (ctypes; argument marshalling only).

Every function here passes device pointers of torch tensors and the current CUDA stream
to libmoe_b200.so; all of the layer's arithmetic runs in that library's CUDA kernels.
There is no fallback: `lib()` raises when the library is missing, and every call raises
MoEError when the library returns an error code.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "moe.h")

MOE_BF16, MOE_FP32 = 0, 1
MOE_COMBINE_FUSED, MOE_COMBINE_DETERMINISTIC = 0, 1

STATUS = {
    0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_ALIGNMENT",
    -4: "MOE_ERR_CUDA", -5: "MOE_ERR_WORKSPACE", -6: "MOE_ERR_DEVICE_CHECK",
    -7: "MOE_ERR_TIMEOUT", -8: "MOE_ERR_NO_DEVICE",
}


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({_status_string(code)})")


class Shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("n_ffn", ctypes.c_int32), ("n_zero", ctypes.c_int32), ("K", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("combine", ctypes.c_int32),
                ("ffn_out_scale", ctypes.c_float)]

    @property
    def E(self) -> int:
        return self.n_ffn + self.n_zero


class Pid(ctypes.Structure):
    _fields_ = [("kp", ctypes.c_float), ("ki", ctypes.c_float), ("kd", ctypes.c_float),
                ("target_ratio", ctypes.c_float)]


def make_shape(T, H, I, n_ffn, n_zero, K, dtype="bf16", combine="fused", ffn_out_scale=1.0):
    dt = {"bf16": MOE_BF16, "fp32": MOE_FP32}[dtype] if isinstance(dtype, str) else int(dtype)
    cb = {"fused": MOE_COMBINE_FUSED, "deterministic": MOE_COMBINE_DETERMINISTIC}[combine] \
        if isinstance(combine, str) else int(combine)
    return Shape(T, H, I, n_ffn, n_zero, K, dt, cb, ffn_out_scale)


def shape_of(cfg, combine="fused", T=None) -> Shape:
    """Shape of a workloads.MoEConfig."""
    return make_shape(cfg.T if T is None else T, cfg.H, cfg.I, cfg.n_ffn, cfg.n_zero, cfg.K,
                      cfg.dtype, combine, cfg.ffn_out_scale)


_P = ctypes.c_void_p
_SZ = ctypes.c_size_t
_SIGS = {
    "moe_scratch_size": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.POINTER(_SZ)]),
    "moe_workspace_size": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.POINTER(_SZ)]),
    "moe_read_device_status": (ctypes.c_int, [_P, _SZ, _P, ctypes.POINTER(ctypes.c_int32)]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_launch_count": (ctypes.c_uint64, []),
    "moe_set_tuning": (ctypes.c_int, [ctypes.c_int, ctypes.c_int64]),
    "moe_get_tuning": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_int64)]),
    "moe_route": (ctypes.c_int, [ctypes.POINTER(Shape)] + [_P] * 11 + [_SZ, _P]),
    "moe_permute": (ctypes.c_int, [ctypes.POINTER(Shape)] + [_P] * 11 + [_SZ, _P]),
    "moe_grouped_ffn": (ctypes.c_int, [ctypes.POINTER(Shape)] + [_P] * 12 + [_SZ, _P]),
    "moe_combine": (ctypes.c_int, [ctypes.POINTER(Shape)] + [_P] * 7 + [_P]),
    "moe_pid_init": (ctypes.c_int, [ctypes.POINTER(Shape), _P, _P, _P]),
    "moe_pid_bias_update": (ctypes.c_int, [ctypes.POINTER(Pid), ctypes.POINTER(Shape)]
                            + [_P] * 6),
    "moe_forward": (ctypes.c_int, [ctypes.POINTER(Shape)] + [_P] * 12 + [_SZ, _P]),
    "moe_permute_static_scratch": (ctypes.c_int, [ctypes.POINTER(Shape)] + [_P] * 10 + [_P]),
    "moe_router_pack": (ctypes.c_int, [ctypes.POINTER(Shape), _P, _P, _P]),
    "moe_route_packed": (ctypes.c_int, [ctypes.POINTER(Shape)] + [_P] * 10 + [_SZ, _P]),
    "moe_lb_loss": (ctypes.c_int, [ctypes.POINTER(Shape)] + [_P] * 5 + [_SZ, _P]),
    "moe_backward_workspace_size": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.POINTER(_SZ)]),
    "moe_backward": (ctypes.c_int, [ctypes.POINTER(Shape)] + [_P] * 19 + [_SZ, _P]),
    "moe_host_pipeline_create": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.POINTER(_P),
                                                 ctypes.POINTER(_P), ctypes.POINTER(_P), _P,
                                                 ctypes.POINTER(_P)]),
    "moe_host_pipeline_submit": (ctypes.c_int, [_P] * 13 + [_SZ]),
    "moe_host_pipeline_join": (ctypes.c_int, [_P]),
    "moe_host_pipeline_destroy": (ctypes.c_int, [_P]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe_b200.so (built by mixture_experts_layer_29_b200.build). Raises if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m mixture_experts_layer_29_b200.build`"
                " (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/moe.h declares."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|uint64_t|const char\*)\s+(moe_\w+)\s*\(", txt,
                                 flags=re.M)))


def _status_string(code: int) -> str:
    try:
        return lib().moe_status_string(code).decode()
    except Exception:  # noqa: BLE001 - message only
        return "?"


def _check(rc: int, where: str):
    if rc != 0:
        raise MoEError(rc, where)


def ptr(t) -> int | None:
    """Device pointer of a tensor (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---- sizes --------------------------------------------------------------------------------

def scratch_size(shape: Shape) -> int:
    n = _SZ(0)
    _check(lib().moe_scratch_size(ctypes.byref(shape), ctypes.byref(n)), "moe_scratch_size")
    return n.value


def workspace_size(shape: Shape) -> int:
    n = _SZ(0)
    _check(lib().moe_workspace_size(ctypes.byref(shape), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def launch_count() -> int:
    return int(lib().moe_launch_count())


# moe_set_tuning switches (include/moe.h): kernel variants with the same results, for
# measurements and tests, and one testing hook
TUNE_PDL, TUNE_GEMM_PAIR, TUNE_PAIR_HALF, TUNE_ROUTER_N = 0, 1, 2, 3
TUNE_ROUTER_MIN_SPLIT, TUNE_BWD_PAIR, TUNE_BWD_DY_ROWS, TUNE_TEST_STALL = 4, 5, 6, 7
TUNE_GATE_UP_BAND, TUNE_DOWN_BAND, TUNE_PAIR_INTERLEAVE, TUNE_PAIR_A_TRIM = 8, 9, 10, 11
TUNE_PAIR_SWAP_AB, TUNE_PAIR_STREAM_HINT, TUNE_PAIR_TAILS, TUNE_PAIR_PREFETCH = 12, 13, 14, 15
TUNE_BWD_WGRAD_GROUP, TUNE_BWD_WGRAD_MIX, TUNE_BWD_WGRAD_BK = 16, 17, 18


def set_tuning(knob: int, value: int):
    _check(lib().moe_set_tuning(int(knob), int(value)), "moe_set_tuning")


def get_tuning(knob: int) -> int:
    v = ctypes.c_int64(0)
    _check(lib().moe_get_tuning(int(knob), ctypes.byref(v)), "moe_get_tuning")
    return int(v.value)


def read_device_status(ws, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(lib().moe_read_device_status(ptr(ws), ws.numel() * ws.element_size(), _stream(stream),
                                        ctypes.byref(v)), "moe_read_device_status")
    return v.value


def _nbytes(ws) -> int:
    return ws.numel() * ws.element_size()


# ---- the steps ----------------------------------------------------------------------------

def route(shape, x, w_router, logits_in, bias, logits_out, topk_idx, topk_gate, counts,
          nffn_hist, zgate, ws, stream=None):
    _check(lib().moe_route(ctypes.byref(shape), ptr(x), ptr(w_router), ptr(logits_in), ptr(bias),
                           ptr(logits_out), ptr(topk_idx), ptr(topk_gate), ptr(counts),
                           ptr(nffn_hist), ptr(zgate), ptr(ws), _nbytes(ws), _stream(stream)),
           "moe_route")


def router_pack(shape, w_router, w_packed, stream=None):
    """Pack the fp32 router weight [E, H] into the exact three-part bf16 form [E, 3H]."""
    _check(lib().moe_router_pack(ctypes.byref(shape), ptr(w_router), ptr(w_packed),
                                 _stream(stream)), "moe_router_pack")


def route_packed(shape, x, w_packed, bias, logits_out, topk_idx, topk_gate, counts, nffn_hist,
                 zgate, ws, stream=None):
    _check(lib().moe_route_packed(ctypes.byref(shape), ptr(x), ptr(w_packed), ptr(bias),
                                  ptr(logits_out), ptr(topk_idx), ptr(topk_gate), ptr(counts),
                                  ptr(nffn_hist), ptr(zgate), ptr(ws), _nbytes(ws),
                                  _stream(stream)), "moe_route_packed")


def permute(shape, topk_idx, topk_gate, zgate, x, offsets, perm_token, row_of, row_gate, x_perm,
            out_acc, ws, stream=None):
    _check(lib().moe_permute(ctypes.byref(shape), ptr(topk_idx), ptr(topk_gate), ptr(zgate),
                             ptr(x), ptr(offsets), ptr(perm_token), ptr(row_of), ptr(row_gate),
                             ptr(x_perm), ptr(out_acc), ptr(ws), _nbytes(ws), _stream(stream)),
           "moe_permute")


def permute_static_scratch(shape, topk_idx, topk_gate, zgate, x, offsets, perm_token, row_of,
                           row_gate, x_perm, out_acc, stream=None):
    """moe_permute without a workspace argument: its scratch is the library's own fixed
    device array (for callers that cannot allocate device memory; see include/moe.h)."""
    _check(lib().moe_permute_static_scratch(ctypes.byref(shape), ptr(topk_idx), ptr(topk_gate),
                                            ptr(zgate), ptr(x), ptr(offsets), ptr(perm_token),
                                            ptr(row_of), ptr(row_gate), ptr(x_perm), ptr(out_acc),
                                            _stream(stream)), "moe_permute_static_scratch")


def grouped_ffn(shape, x, x_perm, offsets, w_gate_up, w_down, perm_token, row_gate, h, y_perm,
                out_acc, ws, stream=None, gu_out=None):
    """x_perm None (bf16): the gate/up GEMM gathers the token rows of x via perm_token.
    gu_out [T*K+128, 2I] bf16: also keep G | U for moe_backward (training forward)."""
    _check(lib().moe_grouped_ffn(ctypes.byref(shape), ptr(x), ptr(x_perm), ptr(offsets),
                                 ptr(w_gate_up), ptr(w_down), ptr(perm_token), ptr(row_gate),
                                 ptr(h), ptr(y_perm), ptr(out_acc), ptr(gu_out), ptr(ws),
                                 _nbytes(ws), _stream(stream)), "moe_grouped_ffn")


def combine(shape, x, y_perm, out_acc, topk_gate, row_of, zgate, out, stream=None):
    _check(lib().moe_combine(ctypes.byref(shape), ptr(x), ptr(y_perm), ptr(out_acc),
                             ptr(topk_gate), ptr(row_of), ptr(zgate), ptr(out), _stream(stream)),
           "moe_combine")


def pid_init(shape, bias, pid_state, stream=None):
    _check(lib().moe_pid_init(ctypes.byref(shape), ptr(bias), ptr(pid_state), _stream(stream)),
           "moe_pid_init")


def pid_bias_update(pid: Pid, shape, counts, nffn_hist, bias, pid_state, stats_out=None,
                    stream=None):
    _check(lib().moe_pid_bias_update(ctypes.byref(pid), ctypes.byref(shape), ptr(counts),
                                     ptr(nffn_hist), ptr(bias), ptr(pid_state), ptr(stats_out),
                                     _stream(stream)), "moe_pid_bias_update")


def backward_workspace_size(shape) -> int:
    n = _SZ(0)
    _check(lib().moe_backward_workspace_size(ctypes.byref(shape), ctypes.byref(n)),
           "moe_backward_workspace_size")
    return n.value


def backward(shape, dout, x, w_router, w_gate_up, w_down, logits, topk_idx, topk_gate, offsets,
             row_of, x_perm, h, y_perm, dx, d_router, d_gate_up, d_down, ws, stream=None,
             gu=None):
    """moe_backward: gradients of the layer for dout, from a deterministic-mode forward;
    gu: G | U saved by grouped_ffn(gu_out=...), or None to recompute them."""
    _check(lib().moe_backward(ctypes.byref(shape), ptr(dout), ptr(x), ptr(w_router),
                              ptr(w_gate_up), ptr(w_down), ptr(logits), ptr(topk_idx),
                              ptr(topk_gate), ptr(offsets), ptr(row_of), ptr(x_perm), ptr(h),
                              ptr(y_perm), ptr(gu), ptr(dx), ptr(d_router), ptr(d_gate_up),
                              ptr(d_down), ptr(ws), _nbytes(ws), _stream(stream)), "moe_backward")


def lb_loss(shape, logits, counts, prob_mean, loss, ws, stream=None):
    """Load-balance loss of the batch (moe_lb_loss): loss [1] fp32, prob_mean [E] or None."""
    _check(lib().moe_lb_loss(ctypes.byref(shape), ptr(logits), ptr(counts), ptr(prob_mean),
                             ptr(loss), ptr(ws), _nbytes(ws), _stream(stream)), "moe_lb_loss")


def forward(shape, x, w_router, logits_in, bias, w_gate_up, w_down, out, topk_idx, topk_gate,
            counts, nffn_hist, ws, stream=None):
    _check(lib().moe_forward(ctypes.byref(shape), ptr(x), ptr(w_router), ptr(logits_in),
                             ptr(bias), ptr(w_gate_up), ptr(w_down), ptr(out), ptr(topk_idx),
                             ptr(topk_gate), ptr(counts), ptr(nffn_hist), ptr(ws), _nbytes(ws),
                             _stream(stream)), "moe_forward")


# ---- buffers for one layer ------------------------------------------------------------------

@dataclass
class StepBuffers:
    """Device buffers of the step-by-step calls for one shape (torch owns the memory)."""
    shape: Shape
    ws: torch.Tensor
    logits: torch.Tensor
    topk_idx: torch.Tensor
    topk_gate: torch.Tensor
    counts: torch.Tensor
    nffn_hist: torch.Tensor
    zgate: torch.Tensor
    offsets: torch.Tensor
    perm_token: torch.Tensor
    row_of: torch.Tensor
    row_gate: torch.Tensor
    x_perm: torch.Tensor
    h: torch.Tensor
    y_perm: torch.Tensor | None
    out_acc: torch.Tensor | None
    out: torch.Tensor

    @staticmethod
    def allocate(shape: Shape, device="cuda") -> "StepBuffers":
        T, H, I, K, E, N = shape.T, shape.H, shape.I, shape.K, shape.E, shape.n_ffn
        dt = torch.bfloat16 if shape.dtype == MOE_BF16 else torch.float32
        rows = T * K + 128
        i32, f32 = torch.int32, torch.float32
        fused = shape.combine == MOE_COMBINE_FUSED
        return StepBuffers(
            shape=shape,
            ws=torch.zeros(max(scratch_size(shape), 256), dtype=torch.uint8, device=device),
            logits=torch.empty(T, E, dtype=f32, device=device),
            topk_idx=torch.empty(T, K, dtype=i32, device=device),
            topk_gate=torch.empty(T, K, dtype=f32, device=device),
            counts=torch.empty(E, dtype=i32, device=device),
            nffn_hist=torch.empty(K + 1, dtype=i32, device=device),
            zgate=torch.empty(max(T, 1), dtype=f32, device=device),
            offsets=torch.empty(N + 1, dtype=i32, device=device),
            perm_token=torch.empty(max(T * K, 1), dtype=i32, device=device),
            row_of=torch.empty(max(T * K, 1), dtype=i32, device=device),
            row_gate=torch.empty(max(T * K, 1), dtype=f32, device=device),
            x_perm=torch.empty(rows, H, dtype=dt, device=device),
            h=torch.empty(rows, I, dtype=dt, device=device),
            y_perm=None if fused else torch.empty(rows, H, dtype=dt, device=device),
            out_acc=torch.empty(max(T, 1), H, dtype=f32, device=device) if fused else None,
            out=torch.empty(max(T, 1), H, dtype=dt, device=device),
        )


def run_steps(b: StepBuffers, x, w_router, logits_in, bias, w_gate_up, w_down, stream=None,
              gather=None, gu_out=None):
    """The layer as its four ABI steps on one stream (moe_route, moe_permute,
    moe_grouped_ffn, moe_combine); returns b.out. gather=True (bf16 only) skips the
    permuted copy of x and lets the gate/up GEMM gather the token rows (less memory,
    slower GEMM). gu_out: keep G | U for moe_backward (a training forward)."""
    s = b.shape
    if gather is None:
        gather = False
    xp = None if gather else b.x_perm
    route(s, x, w_router, logits_in, bias, None if logits_in is not None else b.logits,
          b.topk_idx, b.topk_gate, b.counts, b.nffn_hist, b.zgate, b.ws, stream)
    permute(s, b.topk_idx, b.topk_gate, b.zgate, x, b.offsets, b.perm_token, b.row_of,
            b.row_gate, xp, b.out_acc, b.ws, stream)
    grouped_ffn(s, x, xp, b.offsets, w_gate_up, w_down, b.perm_token, b.row_gate, b.h,
                b.y_perm, b.out_acc, b.ws, stream, gu_out=gu_out)
    combine(s, x, b.y_perm, b.out_acc, b.topk_gate, b.row_of, b.zgate, b.out, stream)
    return b.out


class DenseFFN:
    """A dense SwiGLU FFN, y = W_d (silu(W_g x) * (W_u x)) for every token, on the grouped-FFN
    kernels: moe_grouped_ffn with one group that holds all T tokens (deterministic store,
    so y is written per row). It is the dense FFN a LongCat-Flash layer runs beside its MoE
    (the shortcut-connected MoE overlaps the two).

    forward(x_padded) reads rows [0, T) of x_padded, a [T + 128, H] buffer whose last 128
    rows the GEMM tiles may read but never use; it returns a [T, H] view of y."""

    def __init__(self, T: int, w_gate_up, w_down):
        _, two_i, H = w_gate_up.shape
        self.T, self.H, self.I = T, H, two_i // 2
        assert tuple(w_down.shape) == (1, H, self.I)
        dev = w_gate_up.device
        self.shape = make_shape(T, H, self.I, 1, 0, 1, "bf16", "deterministic")
        self.w_gate_up, self.w_down = w_gate_up, w_down
        self.ws = torch.zeros(max(scratch_size(self.shape), 256), dtype=torch.uint8, device=dev)
        self.offsets = torch.tensor([0, T], dtype=torch.int32, device=dev)
        self.h = torch.empty(T + 128, self.I, dtype=torch.bfloat16, device=dev)
        self.y = torch.empty(T + 128, H, dtype=torch.bfloat16, device=dev)

    def forward(self, x_padded, stream=None):
        assert x_padded.shape[0] >= self.T + 128 and x_padded.shape[1] == self.H
        grouped_ffn(self.shape, x_padded, x_padded, self.offsets, self.w_gate_up, self.w_down,
                    None, None, self.h, self.y, None, self.ws, stream)
        return self.y[: self.T]


class MoELayer:
    """One LongCat-Flash MoE layer on the GPU: weights plus a preallocated workspace.

    forward(x) runs moe_forward (route, permute, grouped SwiGLU FFN, combine) on the
    current stream and returns (out, topk_idx, topk_gate, counts, nffn_hist).
    update_bias() runs one PID step from the last forward's histogram.
    """

    def __init__(self, shape: Shape, w_router, bias, w_gate_up, w_down, pid: Pid | None = None):
        self.shape = shape
        self.w_router, self.bias = w_router, bias
        self.w_gate_up, self.w_down = w_gate_up, w_down
        dev = w_gate_up.device
        self.ws = torch.zeros(workspace_size(shape), dtype=torch.uint8, device=dev)
        T, K, E = shape.T, shape.K, shape.E
        dt = torch.bfloat16 if shape.dtype == MOE_BF16 else torch.float32
        self.out = torch.empty(max(T, 1), shape.H, dtype=dt, device=dev)
        self.topk_idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        self.topk_gate = torch.empty(T, K, dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.nffn_hist = torch.empty(K + 1, dtype=torch.int32, device=dev)
        self.pid = pid
        self.pid_state = torch.empty(3 * shape.n_ffn, dtype=torch.float32, device=dev)
        self.stats = torch.zeros(8, dtype=torch.float32, device=dev)
        pid_init(shape, bias, self.pid_state)

    def forward(self, x, logits_in=None, stream=None):
        forward(self.shape, x, self.w_router, logits_in, self.bias, self.w_gate_up, self.w_down,
                self.out, self.topk_idx, self.topk_gate, self.counts, self.nffn_hist, self.ws,
                stream)
        return self.out, self.topk_idx, self.topk_gate, self.counts, self.nffn_hist

    def update_bias(self, stream=None):
        if self.pid is None:
            raise ValueError("no PID gains given")
        pid_bias_update(self.pid, self.shape, self.counts, self.nffn_hist, self.bias,
                        self.pid_state, self.stats, stream)
        return self.stats

    def forward_host(self, x_host, out_host, logits_in=None, stream=None):
        """End-to-end call from host memory: copy x (pinned) in, run the layer, copy the
        output back into out_host (pinned). Asynchronous on the stream."""
        st = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(st):
            if not hasattr(self, "_x_dev") or self._x_dev.shape != x_host.shape:
                self._x_dev = torch.empty_like(x_host, device=self.out.device)
            self._x_dev.copy_(x_host, non_blocking=True)
            self.forward(self._x_dev, logits_in, st)
            out_host.copy_(self.out[: x_host.shape[0]], non_blocking=True)
        return out_host


class HostPipeline:
    """moe_host_pipeline_*: a layer over batches held in page-locked host memory, each
    batch's copies overlapped with the neighbouring batches' kernels (see include/moe.h).

    Holds the two slots of device staging buffers the C pipeline uses. submit(x_host,
    out_host[, logits_in_host]) queues one batch; join() makes the compute stream wait for
    every queued copy; close() waits for the copies and releases the pipeline."""

    def __init__(self, layer: "MoELayer", with_logits: bool = False, stream=None):
        self.layer = layer
        sh = layer.shape
        dev = layer.out.device
        dt = layer.out.dtype
        self.x = [torch.empty(sh.T, sh.H, dtype=dt, device=dev) for _ in range(2)]
        self.out = [torch.empty(max(sh.T, 1), sh.H, dtype=dt, device=dev) for _ in range(2)]
        self.logits = ([torch.empty(sh.T, sh.E, dtype=torch.float32, device=dev)
                        for _ in range(2)] if with_logits else None)
        arr = _P * 2
        lg = arr(*[ptr(t) for t in self.logits]) if self.logits is not None else None
        self._handle = _P()
        _check(lib().moe_host_pipeline_create(ctypes.byref(sh), arr(*[ptr(t) for t in self.x]),
                                              lg, arr(*[ptr(t) for t in self.out]),
                                              _stream(stream), ctypes.byref(self._handle)),
               "moe_host_pipeline_create")

    def submit(self, x_host, out_host, logits_in_host=None):
        L = self.layer
        _check(lib().moe_host_pipeline_submit(
            self._handle, ptr(x_host), ptr(logits_in_host), ptr(out_host), ptr(L.w_router),
            ptr(L.bias), ptr(L.w_gate_up), ptr(L.w_down), ptr(L.topk_idx), ptr(L.topk_gate),
            ptr(L.counts), ptr(L.nffn_hist), ptr(L.ws), _nbytes(L.ws)),
            "moe_host_pipeline_submit")

    def join(self):
        _check(lib().moe_host_pipeline_join(self._handle), "moe_host_pipeline_join")

    def close(self):
        if getattr(self, "_handle", None) is not None and self._handle.value:
            _check(lib().moe_host_pipeline_destroy(self._handle), "moe_host_pipeline_destroy")
        self._handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass
