"""fp64 CPU oracle for the sparse MoE feed-forward layer (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / reference leg are the only callers.  The
product library never imports, links or runs anything here, and this package
imports nothing from the product package.

Every function mirrors one in ``moe_oracle.c``; the C file's header says
which passage of the pages each one follows.  Parity status: route, layout,
expert FFN and forward are pinned by the ``-m "not gpu"`` tests against the
walkthrough's worked example (yeyulingfeng.com/587419.html section 4), the
closed form of the same section, brute-force top-k and counting sort, a dense
"run every expert then mask" evaluation (llama-cpp-visual-guide lesson 35,
ggml_mul_mat_id section), the E=1/k=1 plain gated MLP, and torch's own SiLU
and tanh-GELU in float64.  The router ahead of the routing (walkthrough
section 3, Gemma4Router) is pinned by the closed form of a constant row, the
unit RMS of the normalised row, exact invariance under power-of-two row
scaling, exact linearity in the scale and the weight, bf16-valued
activations, and a finite zero row.  The FP8 forms (e4m3 codec, per-row
dynamic quantisation, the layer with FP8 experts) are pinned against torch's
float8_e4m3fn conversion, the reconstruction bound of a quantised row, exact
linearity in the w2 scales and a dense float64 restatement.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or \
            os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE",
                               "-fPIC", "-shared", "-fno-fast-math",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int
        lib.oracle_num_threads.restype = i32
        lib.oracle_act.argtypes = [i32, i64, P, P]
        lib.oracle_route.argtypes = [i64, i32, i32, P, P, P, P, P]
        lib.oracle_layout_capacity.argtypes = [i64, i32, i32, i32, i32]
        lib.oracle_layout_capacity.restype = i64
        lib.oracle_layout.argtypes = [i64, i32, i32, i32, i32, P, P, P, i64, P]
        lib.oracle_expert_rows.argtypes = [i32, i32, i32, P, P, P, i64, P, P,
                                           i32, i32, P]
        lib.oracle_forward.argtypes = [i64, i32, i32, i32, i32, i32, i32, i32,
                                       P, P, P, P, P, P, P, P, i64, i32, i32,
                                       P, P, P]
        lib.oracle_router_logits.argtypes = [i64, i32, i32, ctypes.c_double, P, P,
                                             P, P]
        lib.oracle_route_ex.argtypes = [i64, i32, i32, P, P, i32, i32, i32, P, P]
        dbl = ctypes.c_double
        lib.oracle_gemma4_block.argtypes = [i64, i32, i32, i32, i32, i32, i32, P, P, P,
                                            P, P, P, dbl, P, P, dbl, P, P, P, P, P,
                                            i32, P]
        lib.oracle_forward_ex.argtypes = lib.oracle_forward.argtypes + [i32, i32, i32]
        lib.oracle_e4m3_values.argtypes = [i64, P, P]
        lib.oracle_e4m3_codes.argtypes = [i64, P, P]
        lib.oracle_quantize_rows_e4m3.argtypes = [i64, i32, P, P, P]
        lib.oracle_forward_fp8.argtypes = [i64, i32, i32, i32, i32, i32, i32, P, P, P,
                                           P, P, P, P, P, P, P, P, P, i64, i32, P, P, P,
                                           P]
        for f in (lib.oracle_act, lib.oracle_route, lib.oracle_layout,
                  lib.oracle_expert_rows, lib.oracle_forward,
                  lib.oracle_router_logits, lib.oracle_route_ex,
                  lib.oracle_forward_ex, lib.oracle_gemma4_block,
                  lib.oracle_e4m3_values, lib.oracle_e4m3_codes,
                  lib.oracle_quantize_rows_e4m3, lib.oracle_forward_fp8):
            f.restype = i32
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """bf16 torch tensor or uint16 ndarray -> contiguous uint16 ndarray."""
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        return np.ascontiguousarray(a, dtype=np.uint16)
    import torch
    t = a.detach().to("cpu").contiguous()
    assert t.dtype == torch.bfloat16, t.dtype
    return t.view(torch.int16).numpy().view(np.uint16)


def _f32(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    if not isinstance(a, np.ndarray):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=np.float32)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def num_threads() -> int:
    return _load().oracle_num_threads()


def act(kind: int, v) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty_like(v)
    _check(_load().oracle_act(kind, v.size, _ptr(v), _ptr(out)), "act")
    return out


def route(logits, k: int, scale=None, want_probs: bool = False):
    """-> ids [T,k] int32, w [T,k] float64 (and probs [T,E] if asked)."""
    z = _f32(logits)
    T, E = z.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    probs = np.empty((T, E), np.float64) if want_probs else None
    sc = _f32(scale)
    _check(_load().oracle_route(T, E, k, _ptr(z), _ptr(sc), _ptr(ids), _ptr(w),
                                _ptr(probs)), "route")
    return (ids, w, probs) if want_probs else (ids, w)


SCORE_SOFTMAX, SCORE_SIGMOID = 0, 1


def route_ex(logits, k: int, scale=None, scoring: int = SCORE_SOFTMAX,
             n_group: int = 1, topk_group: int = 1):
    """Routing variants (sigmoid scoring, expert groups) -> ids [T,k] int32,
    w [T,k] float64."""
    z = _f32(logits)
    T, E = z.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    sc = _f32(scale)
    _check(_load().oracle_route_ex(T, E, k, _ptr(z), _ptr(sc), scoring, n_group,
                                   topk_group, _ptr(ids), _ptr(w)), "route_ex")
    return ids, w


def layout_capacity(T: int, E: int, k: int, S: int = 0, P: int = 128) -> int:
    return int(_load().oracle_layout_capacity(T, E, k, S, P))


def layout(ids, E: int, S: int = 0, P: int = 128, cap: Optional[int] = None):
    """-> offsets [E+S+1], sorted_slots [cap], slot_row [T,k+S] (int32)."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    if cap is None:
        cap = layout_capacity(T, E, k, S, P)
    offsets = np.empty(E + S + 1, np.int32)
    sorted_slots = np.empty(cap, np.int32)
    slot_row = np.empty((T, k + S), np.int32)
    _check(_load().oracle_layout(T, E, k, S, P, _ptr(ids), _ptr(offsets),
                                 _ptr(sorted_slots), cap, _ptr(slot_row)),
           "layout")
    return offsets, sorted_slots, slot_row


def expert_rows(x, w13, w2, tok, exp_id, act_kind: int, round_h: bool = False,
                nthreads: int = 0) -> np.ndarray:
    """Unweighted FFN outputs y[n,H] of (token, expert) pairs."""
    xu, w13u, w2u = _u16(x), _u16(w13), _u16(w2)
    H = xu.shape[-1]
    I = w2u.shape[-1]
    tok = np.ascontiguousarray(tok, dtype=np.int64)
    exp_id = np.ascontiguousarray(exp_id, dtype=np.int32)
    n = tok.size
    y = np.empty((n, H), np.float64)
    _check(_load().oracle_expert_rows(H, I, act_kind, _ptr(xu), _ptr(w13u),
                                      _ptr(w2u), n, _ptr(tok), _ptr(exp_id),
                                      int(round_h), nthreads, _ptr(y)),
           "expert_rows")
    return y


def router_logits(x, w_router, scale, eps: float) -> np.ndarray:
    """Router logits [T,E] float32 from the bf16 residual [T,H], the bf16
    GateLinear weight [E,H] and the bf16 per-dimension scale [H]."""
    xu, wu, su = _u16(x), _u16(w_router), _u16(scale)
    T, H = xu.shape
    E = wu.shape[0]
    assert wu.shape == (E, H) and su.shape == (H,)
    z = np.empty((T, E), np.float32)
    _check(_load().oracle_router_logits(T, H, E, float(eps), _ptr(xu), _ptr(wu),
                                        _ptr(su), _ptr(z)), "router_logits")
    return z


def forward(x, logits, w13, w2, k: int, act_kind: int, scale=None,
            w13_sh=None, w2_sh=None, tokens=None, round_h: bool = False,
            nthreads: int = 0, scoring: int = SCORE_SOFTMAX, n_group: int = 1,
            topk_group: int = 1):
    """Whole layer in fp64 -> (out [n,H] float64, ids [T,k], w [T,k]).
    scoring / n_group / topk_group select the routing of route_ex."""
    xu, w13u, w2u = _u16(x), _u16(w13), _u16(w2)
    z = _f32(logits)
    T, H = xu.shape
    E = z.shape[1]
    I = w2u.shape[-1]
    sh13, sh2 = _u16(w13_sh), _u16(w2_sh)
    S = 0 if sh13 is None else sh13.shape[0]
    Is = 0 if sh2 is None else sh2.shape[-1]
    tok = None if tokens is None else np.ascontiguousarray(tokens, np.int64)
    n = T if tok is None else tok.size
    out = np.empty((n, H), np.float64)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    sc = _f32(scale)
    _check(_load().oracle_forward_ex(T, H, E, k, I, act_kind, S, Is, _ptr(xu),
                                     _ptr(z), _ptr(sc), _ptr(w13u), _ptr(w2u),
                                     _ptr(sh13), _ptr(sh2), _ptr(tok), n,
                                     int(round_h), nthreads, _ptr(out),
                                     _ptr(ids), _ptr(w), scoring, n_group,
                                     topk_group), "forward")
    return out, ids, w


def gemma4_block(x, norms, eps: float, router_w, router_scale, router_eps: float,
                 w13, w2, scale, mlp_w13, mlp_w2, k: int, act_kind: int,
                 nthreads: int = 0) -> np.ndarray:
    """The MoE block of a Gemma 4 decoder layer from the residual x [T,H]
    bf16 -> the output before its final bf16 rounding, [T,H] float64.
    norms = (pre_ff, post_ff_1, pre_ff_2, post_ff_2, post_ff) gammas [H]
    bf16; mlp_w13 [2*I_dense, H], mlp_w2 [H, I_dense] bf16."""
    xu = _u16(x)
    T, H = xu.shape
    gs = [_u16(g) for g in norms]
    w13u, w2u = _u16(w13), _u16(w2)
    E, I = w13u.shape[0], w2u.shape[-1]
    m13, m2 = _u16(mlp_w13), _u16(mlp_w2)
    Id = m2.shape[-1]
    out = np.empty((T, H), np.float64)
    _check(_load().oracle_gemma4_block(
        T, H, E, k, I, act_kind, Id, _ptr(xu), *[_ptr(g) for g in gs], float(eps),
        _ptr(_u16(router_w)), _ptr(_u16(router_scale)), float(router_eps), _ptr(w13u),
        _ptr(w2u), _ptr(_f32(scale)), _ptr(m13), _ptr(m2), nthreads, _ptr(out)),
        "gemma4_block")
    return out


# ------------------------------------------------------------ FP8 experts

def _u8(a) -> Optional[np.ndarray]:
    """uint8 codes (torch uint8 / float8 tensor or ndarray) -> contiguous uint8."""
    if a is None:
        return None
    if not isinstance(a, np.ndarray):
        import torch
        t = a.detach().to("cpu").contiguous()
        if t.dtype != torch.uint8:
            t = t.view(torch.uint8)
        a = t.numpy()
    return np.ascontiguousarray(a, dtype=np.uint8)


def e4m3_values(codes) -> np.ndarray:
    """Value of every e4m3 code (float64; NaN for 0x7F / 0xFF)."""
    c = _u8(codes)
    out = np.empty(c.shape, np.float64)
    _check(_load().oracle_e4m3_values(c.size, _ptr(c), _ptr(out)), "e4m3_values")
    return out


def e4m3_codes(v) -> np.ndarray:
    """Nearest e4m3 code of each float32 value (ties to even, saturating)."""
    f = _f32(v)
    out = np.empty(f.shape, np.uint8)
    _check(_load().oracle_e4m3_codes(f.size, _ptr(f), _ptr(out)), "e4m3_codes")
    return out


def quantize_rows_e4m3(src):
    """Per-row dynamic e4m3 quantisation of bf16 rows [R, C] -> (codes uint8
    [R, C], scales float32 [R])."""
    su = _u16(src)
    R, C = su.shape
    codes = np.empty((R, C), np.uint8)
    scales = np.empty(R, np.float32)
    _check(_load().oracle_quantize_rows_e4m3(R, C, _ptr(su), _ptr(codes), _ptr(scales)),
           "quantize_rows_e4m3")
    return codes, scales


def forward_fp8(x, logits, w13_q, w13_s, w2_q, w2_s, k: int, act_kind: int, scale=None,
                sh13_q=None, sh13_s=None, sh2_q=None, sh2_s=None, tokens=None,
                nthreads: int = 0, with_slack: bool = False):
    """The layer with FP8 experts in fp64 -> (out [n,H] float64, ids, w),
    and with ``with_slack`` the validity slack [n,H] of every output element
    as a fourth result: how far the admissible other decisions of the
    intermediate's quantisation (bf16 rounding, amax, codes) of an fp32
    implementation can move it.  w13_q [E,2I,H] / w2_q [E,H,I] e4m3 codes with
    per-row fp32 scales w13_s [E,2I] / w2_s [E,H]; shared experts likewise."""
    xu = _u16(x)
    z = _f32(logits)
    T, H = xu.shape
    E = z.shape[1]
    c13, c2 = _u8(w13_q), _u8(w2_q)
    I = c2.shape[-1]
    s13, s2 = _f32(w13_s), _f32(w2_s)
    h13, h2 = _u8(sh13_q), _u8(sh2_q)
    hs13, hs2 = _f32(sh13_s), _f32(sh2_s)
    S = 0 if h13 is None else h13.shape[0]
    tok = None if tokens is None else np.ascontiguousarray(tokens, np.int64)
    n = T if tok is None else tok.size
    out = np.empty((n, H), np.float64)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    slack = np.empty((n, H), np.float64) if with_slack else None
    _check(_load().oracle_forward_fp8(T, H, E, k, I, act_kind, S, _ptr(xu), _ptr(z),
                                      _ptr(_f32(scale)), _ptr(c13), _ptr(s13), _ptr(c2),
                                      _ptr(s2), _ptr(h13), _ptr(hs13), _ptr(h2),
                                      _ptr(hs2), _ptr(tok), n, nthreads, _ptr(out),
                                      _ptr(ids), _ptr(w), _ptr(slack)), "forward_fp8")
    return (out, ids, w, slack) if with_slack else (out, ids, w)
