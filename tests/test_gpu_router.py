"""Parity of the router kernel (moe_router_logits) with the fp64 oracle.

The router ahead of the routing: section 3 of the Gemma 4 walkthrough
("Gemma4Router-MoE 的入口") and the Gemma4Router class of the vLLM page.  Both
sides form the same bf16 activations (RMSNorm in fp32 with the normaliser of
an exact-in-double mean, then the bf16 roundings the page's casts fix); the
logits differ only by the accumulation of the projection, fp32 on the GPU and
double in the oracle.  The bar for that: max|err| <= 3e-4 x RMS(oracle
logits) (fp32 accumulation of H products: relative error ~ sqrt(H/16)
2^-24 times the sum of |products|, a few 1e-5 of the RMS at H = 4096).
Routing on the GPU's logits must then match the oracle's routing of the same
logits bit for bit, and the oracle's routing of its own logits wherever the
k-th and (k+1)-th logits are further apart than the logit error.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_ffn_06_b200 import inputs

pytestmark = pytest.mark.gpu

TOL = 3e-4


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixture_experts_ffn_06_b200 import api as a
    return a


def _case(T, H, E, seed):
    g = torch.Generator().manual_seed(seed)
    return inputs.router_inputs(T, H, E, g, "cpu")


def _gpu_logits(api, x, w, s, eps):
    T, H = x.shape
    E = w.shape[0]
    shape = api.make_shape(T=T, H=H, E=E, k=1, I=8)
    z = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
    api.moe_router_logits(shape, x.cuda(), w.cuda(), s.cuda(), eps, z)
    torch.cuda.synchronize()
    return z.cpu().numpy()


@pytest.mark.parametrize("T,H,E", [
    (64, 256, 8),       # one CTA, Mixtral's E
    (130, 2816, 128),   # ragged token tail, the many-small shape
    (37, 200, 5),       # H not a multiple of 32: a partial 32-column chunk
    (16, 64, 130),      # E > 128: two expert blocks, the second ragged
    (1, 4096, 8),       # one token
    (4, 2816, 128),     # a decode step of the many-small shape
    (13, 200, 5),       # 13 tokens, H = 200
    (16, 1024, 300),    # many expert blocks for one token tile
    (65, 256, 8),       # two token tiles, the second with one token
    (300, 200, 40),     # a ragged token tile and a partial 32-column chunk
    (257, 128, 300),    # many expert blocks, the last one ragged
    (1000, 2048, 64),   # the skewed batch's H and E
    (129, 1024, 256),   # E = 256
    (4096, 4096, 8),    # the Mixtral-shaped batch
])
def test_router_logits_match_oracle(api, T, H, E):
    x, w, s = _case(T, H, E, seed=T + H + E)
    want = oracle.router_logits(x, w, s, 1e-6)
    got = _gpu_logits(api, x, w, s, 1e-6)
    assert np.isfinite(got).all()
    rms = float(np.sqrt(np.mean(want.astype(np.float64) ** 2)))
    err = float(np.abs(got.astype(np.float64) - want).max())
    assert err <= TOL * rms, f"max|err| {err:.3e} > {TOL} x RMS {rms:.3e}"


@pytest.mark.parametrize("T,E", [(8, 8), (20, 8), (150, 32)])
def test_zero_and_constant_rows(api, T, E):
    # all-zero rows stay finite (eps); constant rows normalise to +-1
    x, w, s = _case(T, 128, E, seed=7)
    x[3] = 0.0
    x[5] = 1.5
    want = oracle.router_logits(x, w, s, 1e-6)
    got = _gpu_logits(api, x, w, s, 1e-6)
    assert np.all(got[3] == 0.0)
    rms = float(np.sqrt(np.mean(want.astype(np.float64) ** 2)))
    assert float(np.abs(got - want).max()) <= TOL * rms


@pytest.mark.parametrize("k", [2, 8])
def test_routing_on_router_logits(api, k):
    T, H, E = 200, 2816, 128
    x, w, s = _case(T, H, E, seed=11 + k)
    zo = oracle.router_logits(x, w, s, 1e-6)
    zg = _gpu_logits(api, x, w, s, 1e-6)
    shape = api.make_shape(T=T, H=H, E=E, k=k, I=8)
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, k, dtype=torch.float32, device="cuda")
    api.moe_route(shape, torch.from_numpy(zg).cuda(), None, ids, wt)
    torch.cuda.synchronize()
    ids = ids.cpu().numpy()
    # the same logits: the same decisions, bit for bit
    ref_ids, _ = oracle.route(zg, k)
    assert np.array_equal(ids, ref_ids)
    # the oracle's own logits: the same decisions wherever the k-th and
    # (k+1)-th logits are further apart than the logit error
    own_ids, _ = oracle.route(zo, k)
    srt = -np.sort(-zo.astype(np.float64), axis=1)
    gap = srt[:, k - 1] - srt[:, k]
    rms = float(np.sqrt(np.mean(zo.astype(np.float64) ** 2)))
    clear = gap > 2 * TOL * rms
    assert clear.mean() > 0.9
    assert np.array_equal(np.sort(ids[clear], axis=1), np.sort(own_ids[clear], axis=1))


@pytest.mark.parametrize("path,T", [(1, 37), (2, 4)])  # prefill, decode
def test_forward_from_hidden_states(api, path, T):
    # moe_forward_ex with the router options: logits computed from the
    # residual first.  The oracle runs the layer on the GPU router's own
    # logits (checked against the oracle router above), so both take the
    # same routing decisions; ids bit-exact, output within 2e-2 x RMS.
    from parity_util import assert_out_close, to_device
    shp = inputs.Shape(T=T, H=256, E=8, k=2, I=128, act=1)
    inp = to_device(inputs.make_inputs(shp, seed=3, scale="uniform"))
    g = torch.Generator().manual_seed(5)
    rx, rw, rs = (t.cuda() for t in inputs.router_inputs(T, 256, 8, g, "cpu"))
    s = api.shape_from(shp)
    ws = api.alloc_workspace(s)
    out = torch.empty(T, 256, dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty(T, 256, dtype=torch.float32, device="cuda")
    ids = torch.empty(T, 2, dtype=torch.int32, device="cuda")
    wt = torch.empty(T, 2, dtype=torch.float32, device="cuda")
    api.moe_forward_ex(s, inp.x, None, inp.w13, inp.w2, inp.scale, None, None, out, ws,
                       ids_out=ids, w_out=wt, out_f32=out32, path=path,
                       router=(rx, rw, rs, 1e-6))
    torch.cuda.synchronize()
    assert api.moe_read_error(ws) == 0
    zg = _gpu_logits(api, rx.cpu(), rw.cpu(), rs.cpu(), 1e-6)
    want, ref_ids, ref_w = oracle.forward(inp.x, zg, inp.w13, inp.w2, 2, 1,
                                          scale=inp.scale)
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    assert np.allclose(wt.cpu().numpy(), ref_w, rtol=1e-6, atol=0)
    assert_out_close(out32, want, f"path {path}", bf16=out)
    assert torch.equal(out, out32.to(torch.bfloat16))
