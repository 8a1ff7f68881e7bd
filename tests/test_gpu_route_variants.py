"""Routing variants of llama-cpp-visual-guide lesson 35 on the GPU (sigmoid
scoring, expert groups: a token keeps its best groups, then picks its
experts inside them; the DeepSeek-V3 shape of 256 routed experts, top-8,
one shared expert), through moe_route_ex and moe_forward_ex, against the
fp64 oracle (oracle_route_ex / oracle_forward_ex).

Bars as everywhere: ids and their order bit-exact, gate weights within 1e-6
relative, the fp32 layer output within 2e-2 x RMS of the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_ffn_06_b200 import inputs
from parity_util import (assert_out_close, assert_routing_exact, gpu_forward,
                         oracle_forward, to_device)

pytestmark = pytest.mark.gpu

SOFTMAX, SIGMOID = 0, 1


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixture_experts_ffn_06_b200 import api as a
    return a


def _route_gpu(api, z, k, scale, route):
    T, E = z.shape
    s = api.make_shape(T=T, H=64, E=E, k=k, I=64)
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    api.moe_route_ex(s, z.cuda(), None if scale is None else scale.cuda(), ids, w,
                     route=route)
    torch.cuda.synchronize()
    return ids, w


# (E, k, scoring, n_group, topk_group): DeepSeek-V3 routing; a plain sigmoid
# router; groups of two with padding lanes (E = 40); groups of three whose
# padding entries would index past 32 groups (E = 66); the largest E and k
@pytest.mark.parametrize("E,k,scoring,n_group,topk_group", [
    (256, 8, SIGMOID, 8, 4), (128, 8, SIGMOID, 1, 1), (64, 6, SOFTMAX, 4, 2),
    (40, 5, SOFTMAX, 20, 3), (66, 4, SIGMOID, 22, 2), (512, 32, SIGMOID, 32, 16),
    (8, 2, SOFTMAX, 4, 1)])
def test_route_ex_matches_oracle(api, E, k, scoring, n_group, topk_group):
    gen = torch.Generator().manual_seed(E * 7 + k)
    T = 300
    z = torch.randn(T, E, generator=gen, dtype=torch.float32)
    scale = (0.5 + torch.rand(E, generator=gen)).float()
    route = (scoring, n_group, topk_group)
    ids, w = _route_gpu(api, z, k, scale, route)
    ids_ref, w_ref = oracle.route_ex(z.numpy(), k, scale=scale.numpy(), scoring=scoring,
                                     n_group=n_group, topk_group=topk_group)
    assert_routing_exact(ids, w, ids_ref, w_ref)


@pytest.mark.parametrize("scoring", [SOFTMAX, SIGMOID])
def test_route_ex_ties_between_groups(api, scoring):
    # a handful of values: ties inside groups and between group scores
    gen = torch.Generator().manual_seed(3 + scoring)
    vals = torch.tensor([-1.0, 0.0, 0.5, 0.5, 2.0], dtype=torch.float32)
    z = vals[torch.randint(0, len(vals), (200, 32), generator=gen)]
    route = (scoring, 8, 3)
    ids, w = _route_gpu(api, z, 6, None, route)
    ids_ref, w_ref = oracle.route_ex(z.numpy(), 6, scoring=scoring, n_group=8,
                                     topk_group=3)
    assert_routing_exact(ids, w, ids_ref, w_ref)


CASES = {
    # DeepSeek-V3-shaped routing on small experts: 256 routed experts in 8
    # groups (4 kept), top-8, sigmoid scores, one shared expert
    "deepseek_v3_small": (inputs.Shape(T=6, H=256, E=256, k=8, I=64, act=0,
                                       n_shared=1, I_shared=64), (SIGMOID, 8, 4)),
    "deepseek_v3_T200": (inputs.Shape(T=200, H=256, E=256, k=8, I=64, act=0,
                                      n_shared=1, I_shared=64), (SIGMOID, 8, 4)),
    "grouped_softmax": (inputs.Shape(T=40, H=128, E=16, k=4, I=96, act=1),
                        (SOFTMAX, 4, 2)),
}


@pytest.mark.parametrize("path", [1, 2])
@pytest.mark.parametrize("name", list(CASES))
def test_forward_ex_with_route_variant(api, name, path):
    shp, route = CASES[name]
    inp = inputs.make_inputs(shp, seed=5, scale="uniform")
    want, ids_ref, w_ref = oracle_forward(inp, route=route)
    out, out32, ids, w = gpu_forward(api, to_device(inp), path=path, route=route)
    assert_routing_exact(ids, w, ids_ref, w_ref)
    assert_out_close(out32, want, f"{name} path {path}", bf16=out)
