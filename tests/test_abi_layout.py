"""The Python binding mirrors the C header's structs with ctypes; a field
added on one side only would shift every field after it.  This compiles a
small C program against include/moe.h (gcc, no CUDA needed) and compares
each struct's size and field offsets with the ctypes mirror."""
import ctypes
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FIELDS = {
    "moe_shape": ["T", "H", "E", "k", "I", "n_shared", "I_shared", "act", "pad"],
    "moe_route_opts": ["scoring", "n_group", "topk_group"],
    "moe_forward_opts": ["stage_events", "out_f32", "path", "deterministic", "cta_pairs",
                         "router_x", "router_w", "router_scale", "router_eps", "route"],
    "moe_gemma4_block_params": ["I_dense", "mlp_w13", "mlp_w2", "norm_w", "eps",
                                "router_w", "router_scale", "router_eps"],
    "moe_fp8_experts": ["w13", "w13_scale", "w2", "w2_scale", "w13_sh", "w13_sh_scale",
                        "w2_sh", "w2_sh_scale"],
}


@pytest.fixture(scope="module")
def c_layout(tmp_path_factory):
    d = tmp_path_factory.mktemp("abi")
    src = d / "layout.c"
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "moe.h"',
             "int main(void) {"]
    for st, fields in FIELDS.items():
        lines.append(f'  printf("{st} size %zu\\n", sizeof({st}));')
        for f in fields:
            lines.append(f'  printf("{st} {f} %zu\\n", offsetof({st}, {f}));')
    lines += ["  return 0;", "}"]
    src.write_text("\n".join(lines) + "\n")
    exe = d / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"),
                           "-o", str(exe), str(src)])
    out = subprocess.check_output([str(exe)], text=True)
    table = {}
    for line in out.splitlines():
        st, f, v = line.split()
        table[(st, f)] = int(v)
    return table


def test_ctypes_mirrors_match_the_header(c_layout):
    from mixture_experts_ffn_06_b200 import api
    for st, fields in FIELDS.items():
        cls = getattr(api, st)
        assert ctypes.sizeof(cls) == c_layout[(st, "size")], st
        for f in fields:
            assert getattr(cls, f).offset == c_layout[(st, f)], (st, f)
