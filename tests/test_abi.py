"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function ``include/moe.h`` declares, and
reject bad arguments before it touches the GPU.  Only calls that return
before any CUDA call are made here.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def api():
    from mixture_experts_ffn_06_b200 import build
    build.build()
    from mixture_experts_ffn_06_b200 import api as a
    return a


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[\w\s\*]+?\b(moe_\w+)\s*\(", text,
                                 flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("moe_route", "moe_permute", "moe_expert_ffn", "moe_combine",
                 "moe_forward", "moe_workspace_size", "moe_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol(api):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(api.lib, n), n
    assert set(api.EXPORTS) <= set(names)


def test_nvcc_targets_sm100a():
    from mixture_experts_ffn_06_b200 import build
    flags = " ".join(build.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags


def _shape(api, **kw):
    base = dict(T=64, H=256, E=8, k=2, I=512, act=0, n_shared=0, I_shared=0,
                pad=0)
    base.update(kw)
    return api.make_shape(**base)


def test_capacity_and_workspace_size(api):
    s = _shape(api)
    assert api.moe_layout_capacity(s) == 64 * 2 + 8 * 127
    ws = api.moe_workspace_size(s)
    cap = 64 * 2 + 8 * 127
    assert ws >= cap * 256 * 2 + cap * 512 * 2 + 64 * 256 * 4  # x_perm, h, acc
    sh = _shape(api, n_shared=2, I_shared=512)
    assert api.moe_layout_capacity(sh) == 64 * 2 + 64 * 2 + 10 * 127
    assert api.moe_workspace_size(sh) > ws


@pytest.mark.parametrize("kw,status", [
    (dict(k=9), 1),            # k > E
    (dict(k=0), 1),
    (dict(T=-1), 1),
    (dict(act=7), 1),
    (dict(E=513, k=2), 2),     # above the supported expert count
    (dict(E=64, k=33), 2),
    (dict(H=260), 2),          # rows must be 16-byte multiples
    (dict(I=500), 2),
    (dict(n_shared=1, I_shared=256), 2),
    (dict(pad=64), 2),
    (dict(T=1 << 24), 2),
])
def test_bad_shapes_are_rejected_before_launch(api, kw, status):
    s = _shape(api, **kw)
    assert api.moe_layout_capacity(s) == 0
    assert api.moe_workspace_size(s) == 0
    null = ctypes.c_void_p(0)
    rc = api.lib.moe_route(ctypes.byref(s), null, null, null, null, null)
    assert rc == status
    rc = api.lib.moe_forward(ctypes.byref(s), null, null, null, null, null,
                             null, null, null, null, null, null, 0, null)
    assert rc == status


def test_null_pointers_and_small_workspace(api):
    s = _shape(api)
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: checks come first
    assert api.lib.moe_route(ctypes.byref(s), null, null, null, null, null) == 1
    need = api.moe_workspace_size(s)
    rc = api.lib.moe_permute(ctypes.byref(s), fake, fake, fake, fake, fake,
                             need - 1, null)
    assert rc == 3  # MOE_ERR_WORKSPACE
    rc = api.lib.moe_permute(ctypes.byref(s), fake, fake, fake, fake, null,
                             need, null)
    assert rc == 1
    unaligned = ctypes.c_void_p((1 << 20) + 16)
    rc = api.lib.moe_permute(ctypes.byref(s), fake, fake, fake, fake,
                             unaligned, need, null)
    assert rc == 1
    sh = _shape(api, n_shared=1, I_shared=512)
    rc = api.lib.moe_expert_ffn(ctypes.byref(sh), fake, fake, fake, fake, fake,
                                null, null, fake, fake,
                                api.moe_workspace_size(sh), null)
    assert rc == 1  # shared weights missing
    s1 = _shape(api)
    rc = api.lib.moe_expert_ffn(ctypes.byref(s1), fake, fake, fake, fake, fake,
                                null, null, ctypes.c_void_p((1 << 20) + 8), fake,
                                api.moe_workspace_size(s1), null)
    assert rc == 1  # y_perm not 16-byte aligned


def test_empty_batch_is_a_no_op(api):
    s = _shape(api, T=0)
    null = ctypes.c_void_p(0)
    assert api.lib.moe_route(ctypes.byref(s), null, null, null, null, null) == 0
    assert api.lib.moe_combine(ctypes.byref(s), null, null, null, null,
                               null) == 0


def test_status_strings(api):
    assert api.moe_status_string(0) == "MOE_OK"
    assert api.moe_status_string(5) == "MOE_ERR_TIMEOUT"
    assert api.moe_status_string(99) == "MOE_ERR_UNKNOWN"


def test_router_logits_refuses_bad_arguments(api):
    # rejected on the host before any launch: no GPU needed
    s = api.make_shape(T=4, H=64, E=8, k=1, I=8)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced
    odd = ctypes.c_void_p((1 << 20) + 2)
    null = ctypes.c_void_p(0)
    f = api.lib.moe_router_logits
    assert f(ctypes.byref(s), fake, fake, fake, ctypes.c_float(-1.0), fake, null) == 1
    assert f(ctypes.byref(s), fake, fake, fake, ctypes.c_float(float("inf")), fake, null) == 1
    assert f(ctypes.byref(s), odd, fake, fake, ctypes.c_float(1e-6), fake, null) == 1
    assert f(ctypes.byref(s), null, fake, fake, ctypes.c_float(1e-6), fake, null) == 1
    empty = api.make_shape(T=0, H=64, E=8, k=1, I=8)
    assert f(ctypes.byref(empty), null, null, null, ctypes.c_float(1e-6), null, null) == 0


@pytest.mark.parametrize("opts,status", [
    ((2, 1, 1), 1),      # unknown scoring
    ((0, -1, 1), 1),     # negative group count
    ((1, 3, 1), 1),      # E = 8 is not a multiple of 3 groups
    ((1, 4, 0), 1),      # no group kept
    ((1, 4, 5), 1),      # more groups kept than there are
    ((0, 8, 1), 1),      # one kept group of one expert cannot give k = 2
    ((1, 33, 1), 2),     # above MOE_MAX_GROUPS
])
def test_route_ex_refuses_bad_options(api, opts, status):
    # rejected on the host before any launch: no GPU needed
    s = api.make_shape(T=4, H=64, E=8, k=2, I=8)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced
    ro = api.moe_route_opts(*opts)
    rc = api.lib.moe_route_ex(ctypes.byref(s), fake, fake, ctypes.byref(ro), fake,
                              fake, None)
    assert rc == status
    # the same options reach moe_forward_ex's checks
    fo = api.moe_forward_opts()
    fo.route = ctypes.pointer(ro)
    ws = ctypes.c_void_p(1 << 21)
    rc = api.lib.moe_forward_ex(ctypes.byref(s), fake, fake, fake, fake, fake, None,
                                None, fake, None, None, ws,
                                api.moe_workspace_size(s), ctypes.byref(fo), None)
    assert rc == status


def test_gemma4_block_refuses_bad_arguments(api):
    # rejected on the host before any launch: no GPU needed
    s = api.make_shape(T=4, H=64, E=8, k=2, I=32)
    assert api.moe_gemma4_workspace_size(s, 48) > api.moe_workspace_size(s)
    assert api.moe_gemma4_workspace_size(s, 44) == 0        # I_dense % 8
    sh = api.make_shape(T=4, H=64, E=8, k=2, I=32, n_shared=1, I_shared=32)
    assert api.moe_gemma4_workspace_size(sh, 48) == 0       # no shared experts
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced
    ws = ctypes.c_void_p(1 << 21)
    need = api.moe_gemma4_workspace_size(s, 48)
    prm = api.moe_gemma4_block_params(48, fake.value, fake.value,
                                      (ctypes.c_void_p * 5)(*[1 << 20] * 5), 1e-6,
                                      fake.value, fake.value, 1e-6)
    f = api.lib.moe_gemma4_block
    assert f(ctypes.byref(s), fake, None, fake, fake, None, fake, None, ws, need,
             None) == 1                                      # no params
    assert f(ctypes.byref(s), fake, ctypes.byref(prm), fake, fake, None, fake, None, ws,
             need - 1, None) == 3                            # workspace too small
    prm.norm_w[2] = None
    assert f(ctypes.byref(s), fake, ctypes.byref(prm), fake, fake, None, fake, None, ws,
             need, None) == 1                                # a gamma missing
    assert f(ctypes.byref(sh), fake, ctypes.byref(prm), fake, fake, None, fake, None, ws,
             need, None) == 2                                # shared experts
    prm.norm_w[2] = 1 << 20
    odd = ctypes.c_void_p((1 << 20) + 8)
    assert f(ctypes.byref(s), odd, ctypes.byref(prm), fake, fake, None, fake, None, ws,
             need, None) == 1                                # x not 16-byte aligned
    prm.mlp_w13 = odd.value
    assert f(ctypes.byref(s), fake, ctypes.byref(prm), fake, fake, None, fake, None, ws,
             need, None) == 1                                # a weight not aligned


def test_layer_refuses_unaligned_rows_and_weights(api):
    # rejected on the host before any launch: no GPU needed
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced
    odd = ctypes.c_void_p((1 << 20) + 8)
    null = ctypes.c_void_p(0)
    lib = api.lib
    s = _shape(api)
    need = api.moe_workspace_size(s)
    ws = ctypes.c_void_p(1 << 21)
    fwd = lib.moe_forward_ex
    assert fwd(ctypes.byref(s), fake, fake, odd, fake, null, null, null, fake, null, null,
               ws, need, None, None) == 1                    # w13
    assert fwd(ctypes.byref(s), fake, fake, fake, odd, null, null, null, fake, null, null,
               ws, need, None, None) == 1                    # w2
    assert fwd(ctypes.byref(s), odd, fake, fake, fake, null, null, null, fake, null, null,
               ws, need, None, None) == 1                    # x
    sh = _shape(api, n_shared=1, I_shared=512)
    need_sh = api.moe_workspace_size(sh)
    assert fwd(ctypes.byref(sh), fake, fake, fake, fake, null, odd, fake, fake, null, null,
               ws, need_sh, None, None) == 1                 # a shared expert's w13
    ffn = lib.moe_expert_ffn
    assert ffn(ctypes.byref(s), fake, fake, fake, fake, odd, null, null, fake, ws, need,
               null) == 1                                    # w2
    assert ffn(ctypes.byref(s), odd, fake, fake, fake, fake, null, null, fake, ws, need,
               null) == 1                                    # x


def test_fp8_entry_points_refuse_bad_arguments(api):
    # all rejected on the host before any launch: no GPU needed
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced
    null = ctypes.c_void_p(0)
    lib = api.lib
    # quantiser: cols must be a positive multiple of 8
    assert lib.moe_quantize_rows_e4m3(fake, 4, 12, fake, fake, null) == 1
    assert lib.moe_quantize_rows_e4m3(fake, -1, 16, fake, fake, null) == 1
    assert lib.moe_quantize_rows_e4m3(null, 4, 16, fake, fake, null) == 1
    assert lib.moe_quantize_rows_e4m3(fake, 0, 16, fake, fake, null) == 0  # empty
    s = api.make_shape(T=8, H=64, E=4, k=2, I=64)
    assert api.moe_workspace_size_fp8(s) > api.moe_workspace_size(s)
    w = api.moe_fp8_experts(fake, fake, fake, fake, None, None, None, None)
    opts = api.moe_forward_opts()
    ws_n = api.moe_workspace_size_fp8(s)
    # e4m3 rows need H % 16 == 0 and I % 16 == 0
    s8 = api.make_shape(T=8, H=72, E=4, k=2, I=64)
    assert lib.moe_forward_fp8(ctypes.byref(s8), fake, fake, ctypes.byref(w), None, fake,
                               None, None, fake, 1 << 40, ctypes.byref(opts), null) == 2
    # missing weights, small workspace, the decode path past 64 tokens
    w_bad = api.moe_fp8_experts(fake, None, fake, fake, None, None, None, None)
    assert lib.moe_forward_fp8(ctypes.byref(s), fake, fake, ctypes.byref(w_bad), None,
                               fake, None, None, ctypes.c_void_p(1 << 20), ws_n,
                               ctypes.byref(opts), null) == 1
    assert lib.moe_forward_fp8(ctypes.byref(s), fake, fake, ctypes.byref(w), None, fake,
                               None, None, ctypes.c_void_p(1 << 20), ws_n - 256,
                               ctypes.byref(opts), null) == 3
    # codes and x not 16-byte aligned
    odd = ctypes.c_void_p((1 << 20) + 8)
    w_odd = api.moe_fp8_experts(fake, fake, odd, fake, None, None, None, None)
    assert lib.moe_forward_fp8(ctypes.byref(s), fake, fake, ctypes.byref(w_odd), None,
                               fake, None, None, ctypes.c_void_p(1 << 20), ws_n,
                               ctypes.byref(opts), null) == 1
    assert lib.moe_forward_fp8(ctypes.byref(s), odd, fake, ctypes.byref(w), None, fake,
                               None, None, ctypes.c_void_p(1 << 20), ws_n,
                               ctypes.byref(opts), null) == 1
    dec = api.moe_forward_opts()
    dec.path = api.PATH_DECODE
    s65 = api.make_shape(T=65, H=64, E=4, k=2, I=64)
    assert lib.moe_forward_fp8(ctypes.byref(s65), fake, fake, ctypes.byref(w), None, fake,
                               None, None, ctypes.c_void_p(1 << 20),
                               api.moe_workspace_size_fp8(s65), ctypes.byref(dec), null) == 2
