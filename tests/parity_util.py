"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle on the same seeded inputs."""
import numpy as np
import torch

import oracle
from mixture_experts_ffn_06_b200 import inputs

OUT_TOL = 2e-2      # max |err| <= OUT_TOL * RMS(oracle output)
WEIGHT_RTOL = 1e-6  # gate weights, relative


def to_device(inp: inputs.MoEInputs, device="cuda") -> inputs.MoEInputs:
    def mv(t):
        return None if t is None else t.to(device).contiguous()
    return inputs.MoEInputs(shape=inp.shape, x=mv(inp.x), logits=mv(inp.logits),
                            scale=mv(inp.scale), w13=mv(inp.w13), w2=mv(inp.w2),
                            w13_sh=mv(inp.w13_sh), w2_sh=mv(inp.w2_sh),
                            bias=mv(inp.bias))


def gpu_forward(api, inp: inputs.MoEInputs, with_routing=True, path=0,
                deterministic=False, cta_pairs=0, ws_fill=None, route=None):
    """moe_forward_ex through the C ABI -> (out bf16, out_f32, ids, w).
    Checks that the bf16 output is exactly the round-to-nearest-even of the
    fp32 layer output.  ws_fill: byte written over the workspace past its
    zeroed header before the call (stale contents)."""
    s = api.shape_from(inp.shape)
    T, H, k = inp.shape.T, inp.shape.H, inp.shape.k
    dev = inp.x.device
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    out_f32 = torch.empty(T, H, dtype=torch.float32, device=dev)
    ids = torch.empty(T, k, dtype=torch.int32, device=dev) if with_routing else None
    w = torch.empty(T, k, dtype=torch.float32, device=dev) if with_routing else None
    ws = api.alloc_workspace(s, dev)
    if ws_fill is not None:
        ws[256:].fill_(ws_fill)
    api.moe_forward_ex(s, inp.x, inp.logits, inp.w13, inp.w2, inp.scale,
                       inp.w13_sh, inp.w2_sh, out, ws, ids_out=ids, w_out=w,
                       out_f32=out_f32, path=path, deterministic=deterministic,
                       cta_pairs=cta_pairs, route=route)
    torch.cuda.synchronize()
    assert api.moe_read_error(ws) == 0
    assert torch.equal(out, out_f32.to(torch.bfloat16)), "bf16 rounding step"
    return out, out_f32, ids, w


def oracle_forward(inp: inputs.MoEInputs, tokens=None, route=None):
    scoring, n_group, topk_group = route if route is not None else (0, 1, 1)
    return oracle.forward(inp.x, inp.logits, inp.w13, inp.w2, inp.shape.k,
                          inp.shape.act, scale=inp.scale, w13_sh=inp.w13_sh,
                          w2_sh=inp.w2_sh, tokens=tokens, scoring=scoring,
                          n_group=n_group, topk_group=topk_group)


def assert_out_close(got_t: torch.Tensor, want: np.ndarray, what="",
                     bf16: torch.Tensor = None, slack: np.ndarray = None):
    """Literal bound on the layer output before its final bf16 rounding:
    max|got - want| <= OUT_TOL * RMS(want).  With ``bf16`` (the rounded
    output tensor) that tensor is bounded too, element by element, by
    OUT_TOL * RMS(want) + 2^-8 |want|: the bound plus the largest error a
    rounding to 8 significant bits can add.  ``slack`` (the FP8 layer's
    validity slack from the oracle, per element) widens both bounds by how
    far the admissible other quantisation decisions can move each element."""
    got = got_t.float().cpu().numpy().astype(np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    rms = float(np.sqrt(np.mean(want ** 2)))
    sl = 0.0 if slack is None else slack
    err = float(np.abs(got - want).max())
    excess = np.abs(got - want) - (OUT_TOL * rms + sl)
    assert (excess <= 0).all(), \
        f"{what}: max|err| {err:.3e} > {OUT_TOL} x RMS {rms:.3e}" + \
        ("" if slack is None else f" + slack (by {excess.max():.3e})")
    if bf16 is not None:
        b = bf16.float().cpu().numpy().astype(np.float64)
        assert b.shape == want.shape
        excess = np.abs(b - want) - (OUT_TOL * rms + 2.0 ** -8 * np.abs(want) + sl)
        assert (excess <= 0).all(), \
            f"{what}: bf16 output exceeds the bound by {excess.max():.3e}"
    return err / rms


def assert_routing_exact(ids_gpu, w_gpu, ids_ref, w_ref):
    ids = ids_gpu.cpu().numpy()
    assert (ids == ids_ref).all(), "top-k ids differ"
    w = w_gpu.cpu().numpy().astype(np.float64)
    rel = np.abs(w - w_ref) / np.abs(w_ref)
    assert rel.max() <= WEIGHT_RTOL, f"gate weights rel err {rel.max():.3e}"
