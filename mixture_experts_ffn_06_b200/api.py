"""Python binding of the C ABI in ``include/moe.h`` (argument marshalling only).

Every function has the name of the C entry point it calls and forwards torch
CUDA tensors as raw device pointers on the current torch stream.  Nothing is
computed here: there is no CPU or PyTorch fallback, and importing this module
without the built ``libmoe_b200.so`` raises.  Build it with
``python -m mixture_experts_ffn_06_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT"}
NUM_STAGES = 6
STAGE_NAMES = ("route", "permute", "gather", "w13_gemm_act",
               "w2_gemm_weight_combine", "round_bf16")
EXPORTS = ("moe_layout_capacity", "moe_workspace_size", "moe_router_logits",
           "moe_route",
           "moe_permute", "moe_expert_ffn", "moe_combine", "moe_forward",
           "moe_forward_ex",
           "moe_read_error", "moe_selftest_wait_timeout", "moe_status_string",
           "moe_permute_noalloc", "moe_route_ex", "moe_gemma4_workspace_size",
           "moe_gemma4_block", "moe_quantize_rows_e4m3", "moe_workspace_size_fp8",
           "moe_forward_fp8")


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where} returned {STATUS_NAMES.get(status, status)}")


PATH_AUTO, PATH_PREFILL, PATH_DECODE = 0, 1, 2
DECODE_MAX_T = 16


SCORE_SOFTMAX, SCORE_SIGMOID = 0, 1
MAX_GROUPS = 32


class moe_route_opts(ctypes.Structure):
    _fields_ = [("scoring", ctypes.c_int32), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32)]


class moe_fp8_experts(ctypes.Structure):
    _fields_ = [("w13", ctypes.c_void_p), ("w13_scale", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("w2_scale", ctypes.c_void_p),
                ("w13_sh", ctypes.c_void_p), ("w13_sh_scale", ctypes.c_void_p),
                ("w2_sh", ctypes.c_void_p), ("w2_sh_scale", ctypes.c_void_p)]


class moe_forward_opts(ctypes.Structure):
    _fields_ = [("stage_events", ctypes.c_void_p),
                ("out_f32", ctypes.c_void_p),
                ("path", ctypes.c_int32),
                ("deterministic", ctypes.c_int32),
                ("cta_pairs", ctypes.c_int32),
                ("router_x", ctypes.c_void_p),
                ("router_w", ctypes.c_void_p),
                ("router_scale", ctypes.c_void_p),
                ("router_eps", ctypes.c_float),
                ("route", ctypes.POINTER(moe_route_opts))]


class moe_gemma4_block_params(ctypes.Structure):
    _fields_ = [("I_dense", ctypes.c_int32), ("mlp_w13", ctypes.c_void_p),
                ("mlp_w2", ctypes.c_void_p), ("norm_w", ctypes.c_void_p * 5),
                ("eps", ctypes.c_float), ("router_w", ctypes.c_void_p),
                ("router_scale", ctypes.c_void_p), ("router_eps", ctypes.c_float)]


class moe_shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("I", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("I_shared", ctypes.c_int32), ("act", ctypes.c_int32),
                ("pad", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m mixture_experts_ffn_06_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    P, S = ctypes.c_void_p, ctypes.POINTER(moe_shape)
    st = ctypes.c_int
    lib.moe_layout_capacity.argtypes = [S]
    lib.moe_layout_capacity.restype = ctypes.c_int64
    lib.moe_workspace_size.argtypes = [S]
    lib.moe_workspace_size.restype = ctypes.c_size_t
    lib.moe_router_logits.argtypes = [S, P, P, P, ctypes.c_float, P, P]
    lib.moe_route.argtypes = [S, P, P, P, P, P]
    lib.moe_route_ex.argtypes = [S, P, P, ctypes.POINTER(moe_route_opts), P, P, P]
    lib.moe_permute.argtypes = [S, P, P, P, P, P, ctypes.c_size_t, P]
    lib.moe_expert_ffn.argtypes = [S, P, P, P, P, P, P, P, P, P,
                                   ctypes.c_size_t, P]
    lib.moe_combine.argtypes = [S, P, P, P, P, P]
    lib.moe_forward.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P,
                                ctypes.c_size_t, P]
    lib.moe_forward_ex.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P,
                                   ctypes.c_size_t,
                                   ctypes.POINTER(moe_forward_opts), P]
    lib.moe_read_error.argtypes = [P, ctypes.c_size_t, P]
    lib.moe_gemma4_workspace_size.argtypes = [S, ctypes.c_int32]
    lib.moe_gemma4_workspace_size.restype = ctypes.c_size_t
    lib.moe_gemma4_block.argtypes = [S, P, ctypes.POINTER(moe_gemma4_block_params), P, P,
                                     P, P, P, P, ctypes.c_size_t, P]
    lib.moe_permute_noalloc.argtypes = [S, P, P, P, P, P]
    lib.moe_quantize_rows_e4m3.argtypes = [P, ctypes.c_int64, ctypes.c_int, P, P, P]
    lib.moe_workspace_size_fp8.argtypes = [S]
    lib.moe_workspace_size_fp8.restype = ctypes.c_size_t
    lib.moe_forward_fp8.argtypes = [S, P, P, ctypes.POINTER(moe_fp8_experts), P, P, P, P,
                                    P, ctypes.c_size_t, ctypes.POINTER(moe_forward_opts), P]
    lib.moe_permute_noalloc.restype = st
    lib.moe_selftest_wait_timeout.argtypes = [P, ctypes.c_size_t,
                                              ctypes.c_uint32, P]
    lib.moe_status_string.argtypes = [st]
    lib.moe_status_string.restype = ctypes.c_char_p
    for name in ("moe_router_logits", "moe_route", "moe_route_ex", "moe_permute",
                 "moe_expert_ffn",
                 "moe_combine",
                 "moe_forward", "moe_forward_ex", "moe_read_error", "moe_gemma4_block",
                 "moe_selftest_wait_timeout", "moe_quantize_rows_e4m3", "moe_forward_fp8"):
        getattr(lib, name).restype = st
    return lib


lib = _load()


def make_shape(T: int, H: int, E: int, k: int, I: int, act: int = 0,
               n_shared: int = 0, I_shared: int = 0, pad: int = 0) -> moe_shape:
    return moe_shape(T, H, E, k, I, n_shared, I_shared, act, pad)


def shape_from(s) -> moe_shape:
    """From an ``inputs.Shape`` (or anything with the same attributes)."""
    return make_shape(s.T, s.H, s.E, s.k, s.I, s.act, s.n_shared, s.I_shared)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


def moe_status_string(status: int) -> str:
    return lib.moe_status_string(status).decode()


def moe_layout_capacity(shape: moe_shape) -> int:
    return int(lib.moe_layout_capacity(ctypes.byref(shape)))


def moe_workspace_size(shape: moe_shape) -> int:
    return int(lib.moe_workspace_size(ctypes.byref(shape)))


def alloc_workspace(shape: moe_shape, device="cuda") -> torch.Tensor:
    """Caller-owned workspace (torch allocation), error word zeroed."""
    n = moe_workspace_size(shape)
    if n == 0:
        raise MoEError(1, "moe_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def moe_router_logits(shape, x, w_router, scale, eps, logits, stream=None):
    """Router logits [T,E] fp32 from the bf16 residual x [T,H], the bf16
    GateLinear weight [E,H] and the bf16 per-dimension scale [H]."""
    _check(lib.moe_router_logits(ctypes.byref(shape), _p(x), _p(w_router), _p(scale),
                                 ctypes.c_float(eps), _p(logits), _stream(stream)),
           "moe_router_logits")


def moe_route(shape, logits, scale, ids, w, stream=None):
    _check(lib.moe_route(ctypes.byref(shape), _p(logits), _p(scale), _p(ids),
                         _p(w), _stream(stream)), "moe_route")


def route_opts(route):
    """(scoring, n_group, topk_group) -> moe_route_opts, or None."""
    if route is None:
        return None
    scoring, n_group, topk_group = route
    return moe_route_opts(scoring, n_group, topk_group)


def moe_route_ex(shape, logits, scale, ids, w, route=None, stream=None):
    """Routing variants: ``route`` = (scoring, n_group, topk_group)."""
    ro = route_opts(route)
    _check(lib.moe_route_ex(ctypes.byref(shape), _p(logits), _p(scale),
                            ctypes.byref(ro) if ro is not None else None, _p(ids),
                            _p(w), _stream(stream)), "moe_route_ex")


def moe_permute(shape, ids, offsets, sorted_slots, slot_row, ws, stream=None):
    _check(lib.moe_permute(ctypes.byref(shape), _p(ids), _p(offsets),
                           _p(sorted_slots), _p(slot_row), _p(ws), ws.numel(),
                           _stream(stream)), "moe_permute")


def moe_permute_noalloc(shape, ids, offsets, sorted_slots, slot_row,
                        stream=None):
    """moe_permute without a workspace (scratch in a fixed 1 MiB device array
    inside the library; T*k <= MOE_NOALLOC_MAX_SLOTS; calls must not overlap
    on the GPU)."""
    _check(lib.moe_permute_noalloc(ctypes.byref(shape), _p(ids), _p(offsets),
                                   _p(sorted_slots), _p(slot_row),
                                   _stream(stream)), "moe_permute_noalloc")


def moe_expert_ffn(shape, x, offsets, sorted_slots, w13, w2, w13_sh, w2_sh,
                   y_perm, ws, stream=None):
    _check(lib.moe_expert_ffn(ctypes.byref(shape), _p(x), _p(offsets),
                              _p(sorted_slots), _p(w13), _p(w2), _p(w13_sh),
                              _p(w2_sh), _p(y_perm), _p(ws), ws.numel(),
                              _stream(stream)), "moe_expert_ffn")


def moe_combine(shape, y_perm, slot_row, w, out, stream=None):
    _check(lib.moe_combine(ctypes.byref(shape), _p(y_perm), _p(slot_row), _p(w),
                           _p(out), _stream(stream)), "moe_combine")


def moe_forward(shape, x, logits, w13, w2, scale, w13_sh, w2_sh, out, ws,
                ids_out=None, w_out=None, stream=None):
    _check(lib.moe_forward(ctypes.byref(shape), _p(x), _p(logits), _p(w13),
                           _p(w2), _p(scale), _p(w13_sh), _p(w2_sh), _p(out),
                           _p(ids_out), _p(w_out), _p(ws), ws.numel(),
                           _stream(stream)), "moe_forward")


def moe_forward_ex(shape, x, logits, w13, w2, scale, w13_sh, w2_sh, out, ws,
                   ids_out=None, w_out=None, events=None, out_f32=None,
                   path=PATH_AUTO, deterministic=False, cta_pairs=0,
                   router=None, route=None, stream=None):
    """moe_forward with options: ``events`` (NUM_STAGES + 1 torch.cuda.Event
    created with enable_timing=True, or None to skip one) recorded around
    the stages, ``out_f32``
    ([T,H] fp32) receiving the output before its bf16 rounding, and ``path``
    (PATH_AUTO, PATH_PREFILL or PATH_DECODE); ``deterministic`` selects the
    fixed-order combine on the prefill path; ``cta_pairs`` picks the GEMM
    form (0 auto, 1 single CTAs, 2 CTA pairs); ``router`` = (router_x [T,H],
    router_w [E,H], router_scale [H], eps) computes the logits first
    (``logits`` may then be None); ``route`` = (scoring, n_group,
    topk_group) selects a routing variant (moe_route_ex)."""
    arr = None
    if events is not None:
        if len(events) != NUM_STAGES + 1:
            raise ValueError("need NUM_STAGES + 1 events")
        st = stream if stream is not None else torch.cuda.current_stream()
        for e in events:
            if e is not None and not e.cuda_event:  # torch creates them lazily
                e.record(st)
        arr = (ctypes.c_void_p * (NUM_STAGES + 1))(
            *[ctypes.c_void_p(e.cuda_event if e is not None else 0)
              for e in events])
    rx, rw, rs, reps = router if router is not None else (None, None, None, 0.0)
    ro = route_opts(route)
    opts = moe_forward_opts(
        ctypes.cast(arr, ctypes.c_void_p) if arr is not None else None,
        _p(out_f32), path, int(bool(deterministic)), cta_pairs,
        _p(rx), _p(rw), _p(rs), float(reps),
        ctypes.pointer(ro) if ro is not None else None)
    _check(lib.moe_forward_ex(ctypes.byref(shape), _p(x), _p(logits), _p(w13),
                              _p(w2), _p(scale), _p(w13_sh), _p(w2_sh), _p(out),
                              _p(ids_out), _p(w_out), _p(ws), ws.numel(),
                              ctypes.byref(opts), _stream(stream)),
           "moe_forward_ex")


def moe_read_error(ws, stream=None) -> int:
    """Synchronises the stream; returns (and clears) the workspace error word."""
    return int(lib.moe_read_error(_p(ws), ws.numel(), _stream(stream)))


def moe_selftest_wait_timeout(ws, timeout_us: int, stream=None):
    _check(lib.moe_selftest_wait_timeout(_p(ws), ws.numel(), timeout_us,
                                         _stream(stream)),
           "moe_selftest_wait_timeout")


def moe_gemma4_workspace_size(shape, I_dense: int) -> int:
    return int(lib.moe_gemma4_workspace_size(ctypes.byref(shape), I_dense))


def moe_gemma4_block(shape, x, norms, eps, mlp_w13, mlp_w2, router_w, router_scale,
                     router_eps, w13, w2, scale, out, ws, out_f32=None, stream=None):
    """The Gemma 4 MoE block from the residual x [T,H]: norms = the five
    gammas (pre_ff, post_ff_1, pre_ff_2, post_ff_2, post_ff); mlp_w13
    [2*I_dense, H], mlp_w2 [H, I_dense]; ws of moe_gemma4_workspace_size
    bytes (alloc_gemma4_workspace)."""
    I_dense = int(mlp_w2.shape[-1])
    prm = moe_gemma4_block_params(
        I_dense, _p(mlp_w13), _p(mlp_w2), (ctypes.c_void_p * 5)(*[_p(g) for g in norms]),
        float(eps), _p(router_w), _p(router_scale), float(router_eps))
    _check(lib.moe_gemma4_block(ctypes.byref(shape), _p(x), ctypes.byref(prm), _p(w13),
                                _p(w2), _p(scale), _p(out), _p(out_f32), _p(ws),
                                ws.numel(), _stream(stream)), "moe_gemma4_block")


def alloc_gemma4_workspace(shape, I_dense: int, device="cuda") -> torch.Tensor:
    n = moe_gemma4_workspace_size(shape, I_dense)
    if n == 0:
        raise MoEError(2, "moe_gemma4_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)  # error words zeroed


# ------------------------------------------------------------ FP8 experts

def moe_quantize_rows_e4m3(src, codes, scales, stream=None):
    """Per-row dynamic e4m3 quantisation of bf16 rows src [R, C] into codes
    (uint8 [R, C]) and scales (fp32 [R])."""
    R, C = src.shape
    _check(lib.moe_quantize_rows_e4m3(_p(src), R, C, _p(codes), _p(scales),
                                      _stream(stream)), "moe_quantize_rows_e4m3")


def moe_workspace_size_fp8(shape: moe_shape) -> int:
    return int(lib.moe_workspace_size_fp8(ctypes.byref(shape)))


def alloc_workspace_fp8(shape: moe_shape, device="cuda") -> torch.Tensor:
    n = moe_workspace_size_fp8(shape)
    if n == 0:
        raise MoEError(1, "moe_workspace_size_fp8")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


def fp8_experts(w13, w13_scale, w2, w2_scale, w13_sh=None, w13_sh_scale=None, w2_sh=None,
                w2_sh_scale=None) -> moe_fp8_experts:
    """The weights argument of moe_forward_fp8 (uint8 code tensors, fp32
    row scales)."""
    return moe_fp8_experts(_p(w13), _p(w13_scale), _p(w2), _p(w2_scale), _p(w13_sh),
                           _p(w13_sh_scale), _p(w2_sh), _p(w2_sh_scale))


def moe_forward_fp8(shape, x, logits, weights: moe_fp8_experts, scale, out, ws,
                    ids_out=None, w_out=None, events=None, out_f32=None,
                    path=PATH_AUTO, deterministic=False, cta_pairs=0, router=None,
                    route=None, stream=None):
    """The layer with FP8 experts; ``weights`` from fp8_experts(); the
    options as for moe_forward_ex."""
    arr = None
    if events is not None:
        if len(events) != NUM_STAGES + 1:
            raise ValueError("need NUM_STAGES + 1 events")
        st = stream if stream is not None else torch.cuda.current_stream()
        for e in events:
            if e is not None and not e.cuda_event:
                e.record(st)
        arr = (ctypes.c_void_p * (NUM_STAGES + 1))(
            *[ctypes.c_void_p(e.cuda_event if e is not None else 0) for e in events])
    rx, rw, rs, reps = router if router is not None else (None, None, None, 0.0)
    ro = route_opts(route)
    opts = moe_forward_opts(
        ctypes.cast(arr, ctypes.c_void_p) if arr is not None else None,
        _p(out_f32), path, int(bool(deterministic)), cta_pairs,
        _p(rx), _p(rw), _p(rs), float(reps),
        ctypes.pointer(ro) if ro is not None else None)
    _check(lib.moe_forward_fp8(ctypes.byref(shape), _p(x), _p(logits), ctypes.byref(weights),
                               _p(scale), _p(out), _p(ids_out), _p(w_out), _p(ws),
                               ws.numel(), ctypes.byref(opts), _stream(stream)),
           "moe_forward_fp8")
