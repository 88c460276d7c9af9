"""The C-ABI library without a GPU: it loads, exports every symbol include/moe.h declares,
sizes its workspace, and rejects bad arguments on the host before touching the device."""
import ctypes

import pytest
import torch

from mixture_experts_layer_29_b200 import abi, build
from mixture_experts_layer_29_b200 import workloads as wl


@pytest.fixture(scope="module")
def L():
    build.build()
    return abi.lib()


def test_library_exports_every_declared_function(L):
    names = abi.header_functions()
    assert len(names) == 24
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(abi._SIGS)


def test_tuning_switches_defaults_ranges_and_round_trip(L):
    # every switch starts at its default; the library reads no environment variable
    defaults = {abi.TUNE_PDL: 1, abi.TUNE_GEMM_PAIR: -1, abi.TUNE_PAIR_HALF: 1,
                abi.TUNE_ROUTER_N: 0, abi.TUNE_ROUTER_MIN_SPLIT: 12, abi.TUNE_BWD_PAIR: 1,
                abi.TUNE_BWD_DY_ROWS: 4, abi.TUNE_TEST_STALL: 0, abi.TUNE_GATE_UP_BAND: 0,
                abi.TUNE_DOWN_BAND: 0, abi.TUNE_PAIR_INTERLEAVE: 0, abi.TUNE_PAIR_A_TRIM: 1,
                abi.TUNE_PAIR_SWAP_AB: 1, abi.TUNE_PAIR_STREAM_HINT: 1,
                abi.TUNE_PAIR_TAILS: 0, abi.TUNE_PAIR_PREFETCH: 0,
                abi.TUNE_BWD_WGRAD_GROUP: 16, abi.TUNE_BWD_WGRAD_MIX: 0,
                abi.TUNE_BWD_WGRAD_BK: 64}
    for k, v in defaults.items():
        assert abi.get_tuning(k) == v, k
    bad = [(abi.TUNE_PDL, 2), (abi.TUNE_GEMM_PAIR, -2), (abi.TUNE_ROUTER_N, 128),
           (abi.TUNE_ROUTER_MIN_SPLIT, 0), (abi.TUNE_ROUTER_MIN_SPLIT, 1025),
           (abi.TUNE_BWD_DY_ROWS, 2), (abi.TUNE_BWD_PAIR, 3), (abi.TUNE_TEST_STALL, -1), (abi.TUNE_GATE_UP_BAND, 65),
           (abi.TUNE_DOWN_BAND, -1), (abi.TUNE_PAIR_INTERLEAVE, 2), (abi.TUNE_PAIR_A_TRIM, 3), (abi.TUNE_PAIR_SWAP_AB, 2), (abi.TUNE_PAIR_STREAM_HINT, 5), (abi.TUNE_PAIR_TAILS, 2), (abi.TUNE_PAIR_PREFETCH, 65), (abi.TUNE_BWD_WGRAD_GROUP, 65), (abi.TUNE_BWD_WGRAD_MIX, 65537), (abi.TUNE_BWD_WGRAD_BK, 96), (19, 0), (-1, 0)]
    for k, v in bad:
        assert L.moe_set_tuning(k, v) == -1, (k, v)
    v = ctypes.c_int64(0)
    assert L.moe_get_tuning(19, ctypes.byref(v)) == -1
    assert L.moe_get_tuning(0, None) == -1
    try:
        for k, v in [(abi.TUNE_PDL, 0), (abi.TUNE_GEMM_PAIR, 1), (abi.TUNE_ROUTER_N, 192),
                     (abi.TUNE_ROUTER_MIN_SPLIT, 24), (abi.TUNE_BWD_DY_ROWS, 1),
                     (abi.TUNE_GATE_UP_BAND, 8), (abi.TUNE_DOWN_BAND, 64),
                     (abi.TUNE_PAIR_INTERLEAVE, 1), (abi.TUNE_PAIR_A_TRIM, 0),
                     (abi.TUNE_PAIR_SWAP_AB, 0), (abi.TUNE_PAIR_STREAM_HINT, 0), (abi.TUNE_PAIR_TAILS, 1),
                     (abi.TUNE_PAIR_PREFETCH, 6), (abi.TUNE_BWD_WGRAD_GROUP, 0), (abi.TUNE_BWD_WGRAD_MIX, 512),
                     (abi.TUNE_BWD_WGRAD_BK, 128)]:
            abi.set_tuning(k, v)
            assert abi.get_tuning(k) == v
    finally:
        for k, v in defaults.items():
            abi.set_tuning(k, v)
    for k, v in defaults.items():
        assert abi.get_tuning(k) == v, k


def test_status_strings(L):
    for code in abi.STATUS:
        s = L.moe_status_string(code).decode()
        assert s and s != "unknown status"
    assert L.moe_status_string(12345).decode() == "unknown status"


def _shape(**kw):
    base = dict(T=64, H=256, I=128, n_ffn=16, n_zero=8, K=4, dtype="fp32", combine="fused")
    base.update(kw)
    return abi.make_shape(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(K=25), -1),                       # K > E
    (dict(K=0), -1),
    (dict(T=-1), -1),
    (dict(n_ffn=0), -1),
    (dict(n_ffn=1000, n_zero=100), -2),     # E > 1024
    (dict(n_ffn=100, K=33), -2),            # K > 32
    (dict(H=250), -2),                      # H % 16
    (dict(dtype="bf16", H=192), -2),        # bf16 needs H % 128 == 0
    (dict(dtype="bf16", I=96), -2),         # and I % 128 == 0
    (dict(dtype=7), -1),
    (dict(combine=5), -1),
    (dict(T=1 << 24), -2),
])
def test_shape_limits(L, kw, code):
    n = ctypes.c_size_t(0)
    assert L.moe_workspace_size(ctypes.byref(_shape(**kw)), ctypes.byref(n)) == code
    assert L.moe_scratch_size(ctypes.byref(_shape(**kw)), ctypes.byref(n)) == code


def test_workspace_sizes_cover_the_intermediates(L):
    for name, cfg in wl.CONFIGS.items():
        for comb in ("fused", "deterministic"):
            s = abi.shape_of(cfg, comb)
            scratch, total = abi.scratch_size(s), abi.workspace_size(s)
            esz = 2 if cfg.dtype == "bf16" else 4
            rows = cfg.T * cfg.K + 128
            need = rows * cfg.H * esz + rows * cfg.I * esz + cfg.T * cfg.E * 4
            need += rows * cfg.H * esz if comb == "deterministic" else cfg.T * cfg.H * 4
            assert scratch >= 256 + 2 * cfg.n_ffn * ((cfg.T + 31) // 32) * 4
            assert scratch >= ((cfg.T + 63) // 64) * cfg.E * 8      # load-balance partials
            assert total >= scratch + need, name
    # the full-shape prefill workspace stays a few GB
    s = abi.shape_of(wl.CONFIGS["prefill_bf16"])
    assert abi.workspace_size(s) < 3 * 2**30


def test_host_checks_run_before_any_device_access(L):
    s = _shape()
    p = ctypes.c_void_p
    good = p(1 << 20)
    bad = p((1 << 20) + 4)                   # not 16-byte aligned
    ws_n = abi.scratch_size(s)
    # route: null pointers and misalignment
    args = [good] * 11
    assert L.moe_route(None, *args, ws_n, None) == -1
    a = list(args); a[3] = None              # bias
    assert L.moe_route(ctypes.byref(s), *a, ws_n, None) == -1
    a = list(args); a[4] = bad               # logits_out
    assert L.moe_route(ctypes.byref(s), *a, ws_n, None) == -3
    assert L.moe_route(ctypes.byref(s), *args, ws_n - 1, None) == -5
    # permute / grouped_ffn / forward with a workspace that is too small
    assert L.moe_permute(ctypes.byref(s), *([good] * 11), 16, None) == -5
    assert L.moe_grouped_ffn(ctypes.byref(s), *([good] * 10), None, good, 16, None) == -5
    # gu_out (the training forward's G | U) is for bf16 layers only
    assert L.moe_grouped_ffn(ctypes.byref(s), *([good] * 12), ws_n, None) == -2
    assert L.moe_forward(ctypes.byref(s), *([good] * 12), abi.workspace_size(s) - 1, None) == -5
    # combine: fused mode needs out_acc
    assert L.moe_combine(ctypes.byref(s), good, None, None, None, None, None, good, None) == -1
    # pid: null gains, T = 0
    pid = abi.Pid(0.01, 0.001, 0.0, 8 / 12)
    assert L.moe_pid_bias_update(None, ctypes.byref(s), good, good, good, good, None, None) == -1
    s0 = _shape(T=0)
    assert L.moe_pid_bias_update(ctypes.byref(pid), ctypes.byref(s0), good, good, good, good,
                                 None, None) == -1
    # backward: bf16 only, null pointers, short workspace
    bs = _shape(dtype="bf16", H=256, I=128)
    bw = abi.backward_workspace_size(bs)
    assert L.moe_backward(ctypes.byref(s), *([good] * 19), bw, None) == -2      # fp32 layer
    assert L.moe_backward(ctypes.byref(bs), *([good] * 18), None, bw, None) == -1
    assert L.moe_backward(ctypes.byref(bs), *([good] * 19), bw - 1, None) == -5
    # the saved G | U is optional but must be aligned
    assert L.moe_backward(ctypes.byref(bs), *([good] * 13), bad, *([good] * 5), bw, None) == -3
    # load-balance loss: null counts or loss, unaligned logits, short workspace
    assert L.moe_lb_loss(ctypes.byref(s), good, None, None, good, good, ws_n, None) == -1
    assert L.moe_lb_loss(ctypes.byref(s), good, good, None, None, good, ws_n, None) == -1
    assert L.moe_lb_loss(ctypes.byref(s), bad, good, None, good, good, ws_n, None) == -3
    assert L.moe_lb_loss(ctypes.byref(s), good, good, None, good, good, ws_n - 1, None) == -5
    assert L.moe_read_device_status(None, 256, None, None) == -1


def test_host_pipeline_host_checks(L):
    """moe_host_pipeline_*: argument checks on the host; without a GPU, a valid create
    stops at the device query and keeps nothing."""
    s = _shape(dtype="bf16", H=256, I=128)
    good, bad = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 4)
    arr = ctypes.c_void_p * 2
    two = arr(good, good)
    h = ctypes.c_void_p()
    assert L.moe_host_pipeline_create(ctypes.byref(s), two, None, two, None, None) == -1
    assert L.moe_host_pipeline_create(ctypes.byref(s), None, None, two, None, ctypes.byref(h)) == -1
    assert L.moe_host_pipeline_create(ctypes.byref(s), arr(good, bad), None, two, None,
                                      ctypes.byref(h)) == -3
    assert L.moe_host_pipeline_create(ctypes.byref(s), two, arr(good, None), two, None,
                                      ctypes.byref(h)) == -1
    sk = _shape(dtype="bf16", H=256, I=128, K=25)
    assert L.moe_host_pipeline_create(ctypes.byref(sk), two, None, two, None, ctypes.byref(h)) == -1
    if not torch.cuda.is_available():
        assert L.moe_host_pipeline_create(ctypes.byref(s), two, None, two, None,
                                          ctypes.byref(h)) == -8
        assert not h.value
    assert L.moe_host_pipeline_submit(None, *([good] * 12), 1 << 30) == -1
    assert L.moe_host_pipeline_join(None) == -1
    assert L.moe_host_pipeline_destroy(None) == 0


def test_empty_batch_is_a_no_op(L):
    s = _shape(T=0)
    p = ctypes.c_void_p(1 << 20)
    ws_n = abi.scratch_size(s)
    assert L.moe_route(ctypes.byref(s), *([p] * 11), ws_n, None) == 0
    assert L.moe_permute(ctypes.byref(s), *([p] * 11), ws_n, None) == 0
    assert L.moe_grouped_ffn(ctypes.byref(s), *([p] * 10), None, p, ws_n, None) == 0
    assert L.moe_combine(ctypes.byref(s), *([p] * 7), None) == 0
    assert L.moe_forward(ctypes.byref(s), *([p] * 12), abi.workspace_size(s), None) == 0


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_a_device_reports_no_device(L):
    s = _shape()
    p = ctypes.c_void_p(1 << 20)
    rc = L.moe_route(ctypes.byref(s), *([p] * 11), abi.scratch_size(s), None)
    assert rc == -8
