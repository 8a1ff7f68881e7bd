"""The Gemma 4 MoE block on the GPU (Gemma 4 walkthrough section 1: dense
MLP and MoE in parallel from the same residual, each between its own gamma
RMSNorms, summed unweighted, then the last norm and the residual add),
through moe_gemma4_block, against the fp64 oracle (oracle_gemma4_block).

Bar: the bf16 output is exactly the round-to-nearest-even of the fp32
output, and that fp32 output is within 2e-2 x RMS of the block's update
(out - x) of the oracle plus one bf16 ulp of the element's update,
2^-7 |out - x|.  The last norm returns bf16 by the block's definition, so a
rounding that the fp32 sums upstream decide differently can move an element
by one ulp of that bf16 value (0.031 at magnitudes in [4, 8), 3 % of the
update's RMS): that is the rounding the pages put there, not an error of
the kernels.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_ffn_06_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixture_experts_ffn_06_b200 import api as a
    return a


CASES = {
    # T <= 8: both inner layers take the decode path
    "few_tokens": (inputs.Shape(T=5, H=256, E=16, k=4, I=64, act=1), 96),
    # the prefill path, ragged sizes
    "prefill": (inputs.Shape(T=70, H=200, E=8, k=2, I=104, act=0), 136),
    # the 26B-A4B shapes: H=2816, 128 experts of I=704, top-8, dense I=2112
    "gemma4_26b_shapes": (inputs.Shape(T=16, H=2816, E=128, k=8, I=704, act=1), 2112),
}


@pytest.mark.parametrize("name", list(CASES))
def test_block_matches_oracle(api, name):
    shp, Id = CASES[name]
    moe = inputs.make_inputs(shp, seed=1, scale="uniform")
    blk = inputs.gemma4_block_inputs(shp.T, shp.H, shp.E, Id, seed=2)
    want = oracle.gemma4_block(blk.x, blk.norms, 1e-6, blk.router_w, blk.router_scale,
                               1e-6, moe.w13, moe.w2, moe.scale, blk.mlp_w13, blk.mlp_w2,
                               shp.k, shp.act)
    c = lambda t: t.cuda().contiguous()  # noqa: E731
    s = api.shape_from(shp)
    out = torch.empty(shp.T, shp.H, dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty(shp.T, shp.H, dtype=torch.float32, device="cuda")
    ws = api.alloc_gemma4_workspace(s, Id)
    api.moe_gemma4_block(s, c(blk.x), [c(g) for g in blk.norms], 1e-6, c(blk.mlp_w13),
                         c(blk.mlp_w2), c(blk.router_w), c(blk.router_scale), 1e-6,
                         c(moe.w13), c(moe.w2), c(moe.scale), out, ws, out_f32=out32)
    torch.cuda.synchronize()
    assert torch.equal(out, out32.to(torch.bfloat16))
    got = out32.cpu().numpy().astype(np.float64)
    x = blk.x.float().numpy().astype(np.float64)
    upd = float(np.sqrt(np.mean((want - x) ** 2)))
    assert np.isfinite(got).all()
    bound = 2e-2 * upd + 2.0 ** -7 * np.abs(want - x)
    excess = np.abs(got - want) - bound
    assert excess.max() <= 0, (f"max|err| {np.abs(got - want).max():.3e}, update RMS "
                               f"{upd:.3e}, worst excess {excess.max():.3e}")


def _block_args(api, shp, moe, blk):
    """moe_gemma4_block's arguments up to ``out``, on the device."""
    c = lambda t: t.cuda().contiguous()  # noqa: E731
    s = api.shape_from(shp)
    args = (s, c(blk.x), [c(g) for g in blk.norms], 1e-6, c(blk.mlp_w13), c(blk.mlp_w2),
            c(blk.router_w), c(blk.router_scale), 1e-6, c(moe.w13), c(moe.w2),
            c(moe.scale))
    return args


def test_block_branches_join_on_the_callers_stream(api):
    """The dense MLP runs on a second stream; the call must still be
    complete once the caller's stream alone is synchronised, and the
    block's error word (moe_read_error on its workspace) is clear."""
    shp, Id = CASES["gemma4_26b_shapes"]
    moe = inputs.make_inputs(shp, seed=3, scale="uniform")
    blk = inputs.gemma4_block_inputs(shp.T, shp.H, shp.E, Id, seed=4)
    args = _block_args(api, shp, moe, blk)
    s = args[0]
    ws = api.alloc_gemma4_workspace(s, Id)
    ref = torch.empty(shp.T, shp.H, dtype=torch.bfloat16, device="cuda")
    api.moe_gemma4_block(*args, ref, ws)
    torch.cuda.synchronize()
    st = torch.cuda.Stream()
    for _ in range(3):
        out = torch.full((shp.T, shp.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        torch.cuda.current_stream().synchronize()
        with torch.cuda.stream(st):
            api.moe_gemma4_block(*args, out, ws, stream=st)
        st.synchronize()  # the caller's stream only
        assert torch.equal(out, ref)
    assert api.moe_read_error(ws) == 0


def test_block_captured_in_a_cuda_graph(api):
    """The fork onto the second stream and the join back are events, so the
    call captures into one graph; replays give the eager result bit for bit
    (both inner layers take the deterministic decode path here)."""
    shp, Id = CASES["few_tokens"]
    moe = inputs.make_inputs(shp, seed=5, scale="uniform")
    blk = inputs.gemma4_block_inputs(shp.T, shp.H, shp.E, Id, seed=6)
    args = _block_args(api, shp, moe, blk)
    s = args[0]
    ws = api.alloc_gemma4_workspace(s, Id)
    ref = torch.empty(shp.T, shp.H, dtype=torch.bfloat16, device="cuda")
    api.moe_gemma4_block(*args, ref, ws)
    torch.cuda.synchronize()
    out = torch.zeros(shp.T, shp.H, dtype=torch.bfloat16, device="cuda")
    st = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(st):
        api.moe_gemma4_block(*args, out, ws, stream=st)  # warm-up outside capture
    st.synchronize()
    out.zero_()
    with torch.cuda.graph(g, stream=st):
        api.moe_gemma4_block(*args, out, ws, stream=st)
    for _ in range(2):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    del g
    assert api.moe_read_error(ws) == 0
