"""Parity of the layer with FP8 (e4m3) experts on the GPU with the fp64
oracle (through the C ABI).

Per-expert FP8 checkpoints (the sglang PR on Gemma 4 FP8 per-expert
loading; load_weights on the vLLM API page) carry a weight_scale per
weight; the reading is one fp32 scale per output row, activations and the
bf16 intermediate quantised per row at run time.  Bars: the row quantiser's
codes and scales bit-exact (IEEE fp32 steps on both sides); routing ids
bit-exact and gate weights within 1e-6 relative; the layer output within
2e-2 x RMS(oracle) + slack on the fp32 result, the bf16 output its exact
rounding and within 2e-2 x RMS + 2^-8 |oracle| + slack.  The slack (from
the oracle, per element) is how far the quantisation decisions on the
intermediate that an fp32 computation of it may take either way (a value
within its rounding error of a bf16 or e4m3 boundary, or of the row's amax)
can move the element; it is zero where no such decision exists.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_ffn_06_b200 import inputs
from parity_util import assert_out_close, assert_routing_exact

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixture_experts_ffn_06_b200 import api as a
    return a


@pytest.mark.parametrize("R,C", [(1, 8), (37, 104), (300, 2816), (64, 4096)])
def test_quantize_rows_bit_exact(api, R, C):
    g = torch.Generator().manual_seed(R + C)
    x = torch.randn(R, C, generator=g) * torch.exp(torch.randn(R, 1, generator=g) * 3)
    if R > 2:
        x[1] = 0.0                      # all-zero row: scale 1
        x[2, 5] = 3e4                   # one large value sets the scale
        x[2, 6] = -2e-30                # tiny values flush to (signed) zero
    xb = x.to(torch.bfloat16)
    codes = torch.empty(R, C, dtype=torch.uint8, device="cuda")
    scales = torch.empty(R, dtype=torch.float32, device="cuda")
    api.moe_quantize_rows_e4m3(xb.cuda(), codes, scales)
    torch.cuda.synchronize()
    want_c, want_s = oracle.quantize_rows_e4m3(xb)
    assert np.array_equal(scales.cpu().numpy(), want_s)
    assert np.array_equal(codes.cpu().numpy(), want_c)


def _to(t):
    return None if t is None else t.cuda().contiguous()


def _gpu_fp8(api, inp, fp, det=False, pairs=0, path=0):
    shp = inp.shape
    s = api.shape_from(shp)
    T, H, k = shp.T, shp.H, shp.k
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty(T, H, dtype=torch.float32, device="cuda")
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    ws = api.alloc_workspace_fp8(s)
    wts = [_to(t) for t in (fp.w13_q, fp.w13_s, fp.w2_q, fp.w2_s, fp.sh13_q, fp.sh13_s,
                            fp.sh2_q, fp.sh2_s)]
    weights = api.fp8_experts(*wts)
    api.moe_forward_fp8(s, _to(inp.x), _to(inp.logits), weights, _to(inp.scale), out, ws,
                        ids_out=ids, w_out=w, out_f32=out32, deterministic=det,
                        cta_pairs=pairs, path=path)
    torch.cuda.synchronize()
    assert api.moe_read_error(ws) == 0
    assert torch.equal(out, out32.to(torch.bfloat16)), "bf16 rounding step"
    return out, out32, ids, w


def _oracle_fp8(inp, fp, tokens=None):
    """-> (out, ids, w, slack)"""
    return oracle.forward_fp8(inp.x, inp.logits, fp.w13_q, fp.w13_s, fp.w2_q, fp.w2_s,
                              k=inp.shape.k, act_kind=inp.shape.act, scale=inp.scale,
                              sh13_q=fp.sh13_q, sh13_s=fp.sh13_s, sh2_q=fp.sh2_q,
                              sh2_s=fp.sh2_s, tokens=tokens, with_slack=True)


SHAPES = {
    "tiny": inputs.Shape(T=64, H=256, E=8, k=2, I=512),
    "ragged": inputs.Shape(T=37, H=208, E=5, k=3, I=112, act=1),  # K, N tails
    "shared": inputs.Shape(T=40, H=128, E=6, k=2, I=96, n_shared=2, I_shared=96),
    "one_token": inputs.Shape(T=1, H=128, E=8, k=2, I=128),
    "gemma_T130": inputs.Shape(T=130, H=2816, E=128, k=8, I=704, act=1),  # narrow tiles
    "pairs": inputs.Shape(T=700, H=208, E=3, k=2, I=112, act=1),
    "pairs_wide_I": inputs.Shape(T=600, H=128, E=2, k=2, I=1024),
    "few_shared": inputs.Shape(T=3, H=208, E=6, k=2, I=96, n_shared=2, I_shared=96),
}
VARIANTS = {"fast": (False, 0), "det": (True, 0), "pairs": (False, 2)}


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("name", list(SHAPES))
def test_forward_fp8_every_element(api, name, variant):
    shp = SHAPES[name]
    inp = inputs.make_inputs(shp, seed=4, scale="uniform")
    fp = inputs.fp8_experts(shp, seed=104)
    want, ids_ref, w_ref, slack = _oracle_fp8(inp, fp)
    det, pairs = VARIANTS[variant]
    out, out32, ids, w = _gpu_fp8(api, inp, fp, det=det, pairs=pairs)
    assert_routing_exact(ids, w, ids_ref, w_ref)
    assert_out_close(out32, want, f"{name} fp8 ({variant})", bf16=out, slack=slack)


DECODE_SHAPES = {
    "one_token": SHAPES["one_token"],                        # N = 16
    "few": inputs.Shape(T=5, H=208, E=5, k=3, I=112, act=1),  # K and row tails
    "few_shared": SHAPES["few_shared"],                      # 2 shared experts, T = 3
    "eight": inputs.Shape(T=8, H=1024, E=16, k=4, I=320),    # N = 16
    "nine": inputs.Shape(T=9, H=1024, E=16, k=4, I=320),     # N = 16
    "gemma_T16": inputs.Shape(T=16, H=2816, E=128, k=8, I=704, act=1),
    "ragged": SHAPES["ragged"],                              # N = 64, T = 37
    "shared": SHAPES["shared"],                              # 2 shared experts
    "T64": inputs.Shape(T=64, H=256, E=8, k=2, I=128),       # N = 64, split units
}


@pytest.mark.parametrize("name", list(DECODE_SHAPES))
def test_forward_fp8_decode_path_every_element(api, name):
    """The decode path's tensor-core form with e4m3 weights: x and each
    (expert, token) row of h quantised per row, the scales applied after the
    split units' fixed-order reduction."""
    shp = DECODE_SHAPES[name]
    inp = inputs.make_inputs(shp, seed=10, scale="uniform")
    fp = inputs.fp8_experts(shp, seed=110)
    want, ids_ref, w_ref, slack = _oracle_fp8(inp, fp)
    out, out32, ids, w = _gpu_fp8(api, inp, fp, path=api.PATH_DECODE)
    assert_routing_exact(ids, w, ids_ref, w_ref)
    assert_out_close(out32, want, f"{name} fp8 decode", bf16=out, slack=slack)


@pytest.mark.parametrize("name", ["decode_t1", "decode_t4", "decode_t16", "decode_t64"])
def test_forward_fp8_decode_sweep_every_element(api, name):
    """The decode sweep's shapes (H=2816, E=128, k=8, I=704, tanh-GELU) with
    FP8 experts, on the path the layer picks by itself: the tensor-core
    decode form up to 16 tokens, the prefill GEMMs above.  Every output
    element against the oracle."""
    shp = inputs.shape_of(name)
    inp = inputs.make_inputs(name, seed=0, device="cuda")
    fp = inputs.fp8_experts(shp, seed=1, device="cuda")
    out, out32, ids, w = _gpu_fp8(api, inp, fp)
    want, ids_ref, w_ref, slack = _oracle_fp8(inp, fp)
    assert_routing_exact(ids, w, ids_ref, w_ref)
    assert_out_close(out32, want, f"{name} fp8", bf16=out, slack=slack)


@pytest.mark.parametrize("name", ["gemma_T16", "eight"])
def test_forward_fp8_decode_path_is_deterministic(api, name):
    shp = DECODE_SHAPES[name]
    inp = inputs.make_inputs(shp, seed=11, scale="uniform")
    fp = inputs.fp8_experts(shp, seed=111)
    a = _gpu_fp8(api, inp, fp, path=api.PATH_DECODE)
    b = _gpu_fp8(api, inp, fp, path=api.PATH_DECODE)
    assert torch.equal(a[1], b[1])


def test_forward_fp8_refuses_the_decode_path_past_64_tokens(api):
    shp = inputs.Shape(T=65, H=128, E=8, k=2, I=128)
    inp = inputs.make_inputs(shp, seed=1)
    fp = inputs.fp8_experts(shp, seed=2)
    with pytest.raises(api.MoEError) as e:
        _gpu_fp8(api, inp, fp, path=api.PATH_DECODE)
    assert e.value.status == 2


def test_forward_fp8_deterministic_repeats_bit_for_bit(api):
    shp = SHAPES["gemma_T130"]
    inp = inputs.make_inputs(shp, seed=5, scale="uniform")
    fp = inputs.fp8_experts(shp, seed=105)
    a = _gpu_fp8(api, inp, fp, det=True)
    b = _gpu_fp8(api, inp, fp, det=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_forward_fp8_full_size_many_small(api):
    """The many-small-experts prefill (T=8192, H=2816, E=128, k=8, I=704,
    tanh-GELU) with FP8 experts: every routing decision, and the outputs of
    one token from every 128-row (expert, m-tile) of the layout."""
    shp = inputs.shape_of("many_small_prefill")
    inp = inputs.make_inputs("many_small_prefill", seed=0, device="cuda")
    fp = inputs.fp8_experts(shp, seed=1, device="cuda")
    out, out32, ids, w = _gpu_fp8(api, inp, fp)
    ids_ref, w_ref = oracle.route(inp.logits, shp.k, scale=inp.scale)
    assert_routing_exact(ids, w, ids_ref, w_ref)
    offsets, sorted_slots, _ = oracle.layout(ids_ref, shp.E, 0, 128)
    rng = np.random.default_rng(3)
    tok = {0, shp.T - 1}
    for g in range(shp.E):
        for r0 in range(int(offsets[g]), int(offsets[g + 1]), 128):
            rows = sorted_slots[r0:r0 + 128]
            real = rows[rows >= 0]
            if real.size:
                tok.add(int(real[rng.integers(real.size)]) // shp.k)
    tok = np.array(sorted(tok), np.int64)
    want, _, _, slack = _oracle_fp8(inp, fp, tokens=tok)
    sel = torch.from_numpy(tok).cuda()
    assert_out_close(out32[sel], want, f"many-small fp8, {len(tok)} tokens",
                     bf16=out[sel], slack=slack)


# ---------------------------------------------------------------- integrity

BAND = 4096      # guard bytes on each side of a buffer
PATTERN = 0xA5


class _Guarded:
    """A buffer inside an allocation whose BAND bytes on either side hold
    PATTERN."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.n = n
        self.raw = torch.full((BAND + n + BAND,), PATTERN, dtype=torch.uint8,
                              device="cuda")
        self.t = self.raw[BAND:BAND + n].view(dtype).view(*shape)

    def intact(self) -> bool:
        torch.cuda.synchronize()
        return bool((self.raw[:BAND] == PATTERN).all()) and \
            bool((self.raw[BAND + self.n:] == PATTERN).all())


@pytest.mark.parametrize("variant", list(VARIANTS) + ["decode"])
@pytest.mark.parametrize("name", ["ragged", "shared", "gemma_T130", "pairs", "few_shared"])
def test_forward_fp8_writes_only_its_buffers(api, name, variant):
    shp = SHAPES[name]
    inp = inputs.make_inputs(shp, seed=6, scale="uniform")
    fp = inputs.fp8_experts(shp, seed=106)
    s = api.shape_from(shp)
    T, H, k = shp.T, shp.H, shp.k
    out = _Guarded((T, H), torch.bfloat16)
    out32 = _Guarded((T, H), torch.float32)
    ids = _Guarded((T, k), torch.int32)
    w = _Guarded((T, k), torch.float32)
    ws = _Guarded((api.moe_workspace_size_fp8(s),), torch.uint8)
    ws.t[:256].zero_()
    wts = [_to(t) for t in (fp.w13_q, fp.w13_s, fp.w2_q, fp.w2_s, fp.sh13_q, fp.sh13_s,
                            fp.sh2_q, fp.sh2_s)]
    if variant == "decode" and T > 64:
        pytest.skip("the decode path takes FP8 experts up to 64 tokens")
    det, pairs = VARIANTS.get(variant, (False, 0))
    path = api.PATH_DECODE if variant == "decode" else 0
    for _ in range(2):  # the second call finds the first call's workspace
        api.moe_forward_fp8(s, _to(inp.x), _to(inp.logits), api.fp8_experts(*wts),
                            _to(inp.scale), out.t, ws.t, ids_out=ids.t, w_out=w.t,
                            out_f32=out32.t, deterministic=det, cta_pairs=pairs,
                            path=path)
    assert api.moe_read_error(ws.t) == 0
    assert torch.isfinite(out32.t).all()
    for nm, g in (("out", out), ("out_f32", out32), ("ids", ids), ("w", w),
                  ("workspace", ws)):
        assert g.intact(), f"{nm}: a guard band was overwritten"


@pytest.mark.parametrize("name", ["gemma_T130", "few_shared"])
def test_forward_fp8_stale_workspace_changes_nothing(api, name):
    """A workspace full of 0xFF bytes (NaN in bf16 and fp32, -1 as an index)
    past its zeroed header gives the same bits as a clean one (fixed-order
    combine; the decode path at 3 tokens)."""
    shp = SHAPES[name]
    inp = inputs.make_inputs(shp, seed=7, scale="uniform")
    fp = inputs.fp8_experts(shp, seed=107)
    s = api.shape_from(shp)
    wts = [_to(t) for t in (fp.w13_q, fp.w13_s, fp.w2_q, fp.w2_s, fp.sh13_q, fp.sh13_s,
                            fp.sh2_q, fp.sh2_s)]
    outs = []
    for fill in (None, 0xFF):
        ws = api.alloc_workspace_fp8(s)
        if fill is not None:
            ws[256:].fill_(fill)
        out32 = torch.empty(shp.T, shp.H, dtype=torch.float32, device="cuda")
        out = torch.empty(shp.T, shp.H, dtype=torch.bfloat16, device="cuda")
        api.moe_forward_fp8(s, _to(inp.x), _to(inp.logits), api.fp8_experts(*wts),
                            _to(inp.scale), out, ws, out_f32=out32, deterministic=True)
        torch.cuda.synchronize()
        assert api.moe_read_error(ws) == 0
        outs.append(out32)
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("name", ["shared", "few_shared"])
def test_forward_fp8_captured_in_a_cuda_graph(api, name):
    """One graph of the FP8 layer (fixed-order combine; the decode path at 3
    tokens) replays the eager result bit for bit."""
    shp = SHAPES[name]
    inp = inputs.make_inputs(shp, seed=8, scale="uniform")
    fp = inputs.fp8_experts(shp, seed=108)
    s = api.shape_from(shp)
    wts = [_to(t) for t in (fp.w13_q, fp.w13_s, fp.w2_q, fp.w2_s, fp.sh13_q, fp.sh13_s,
                            fp.sh2_q, fp.sh2_s)]
    weights = api.fp8_experts(*wts)
    x, z, sc = _to(inp.x), _to(inp.logits), _to(inp.scale)
    ws = api.alloc_workspace_fp8(s)
    ref = torch.empty(shp.T, shp.H, dtype=torch.float32, device="cuda")
    out = torch.empty(shp.T, shp.H, dtype=torch.bfloat16, device="cuda")
    api.moe_forward_fp8(s, x, z, weights, sc, out, ws, out_f32=ref, deterministic=True)
    torch.cuda.synchronize()
    got = torch.zeros_like(ref)
    st = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        api.moe_forward_fp8(s, x, z, weights, sc, out, ws, out_f32=got, deterministic=True,
                            stream=st)
    for _ in range(2):
        got.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(got, ref)
    del g
    assert api.moe_read_error(ws) == 0


def test_forward_fp8_from_hidden_states(api):
    """moe_forward_fp8 with the router options: the logits come from the
    residual first.  The oracle runs the FP8 layer on the GPU router's own
    logits (moe_router_logits, checked against the oracle's router in the
    router tests), so both take the same routing decisions."""
    from parity_util import assert_routing_exact
    shp = SHAPES["ragged"]
    T, H, E = shp.T, shp.H, shp.E
    inp = inputs.make_inputs(shp, seed=9, scale="uniform")
    fp = inputs.fp8_experts(shp, seed=109)
    g = torch.Generator().manual_seed(19)
    rx, rw, rs = (t.cuda() for t in inputs.router_inputs(T, H, E, g, "cpu"))
    s = api.shape_from(shp)
    ws = api.alloc_workspace_fp8(s)
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    out32 = torch.empty(T, H, dtype=torch.float32, device="cuda")
    ids = torch.empty(T, shp.k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, shp.k, dtype=torch.float32, device="cuda")
    wts = [_to(t) for t in (fp.w13_q, fp.w13_s, fp.w2_q, fp.w2_s)]
    api.moe_forward_fp8(s, _to(inp.x), None, api.fp8_experts(*wts), _to(inp.scale), out,
                        ws, ids_out=ids, w_out=w, out_f32=out32, router=(rx, rw, rs, 1e-6))
    zg = torch.empty(T, E, dtype=torch.float32, device="cuda")
    api.moe_router_logits(s, rx, rw, rs, 1e-6, zg)
    torch.cuda.synchronize()
    assert api.moe_read_error(ws) == 0
    zg = zg.cpu().numpy()
    want, ids_ref, w_ref, slack = oracle.forward_fp8(
        inp.x, zg, fp.w13_q, fp.w13_s, fp.w2_q, fp.w2_s, k=shp.k, act_kind=shp.act,
        scale=inp.scale, with_slack=True)
    assert_routing_exact(ids, w, ids_ref, w_ref)
    assert_out_close(out32, want, "fp8 from hidden states", bf16=out, slack=slack)
