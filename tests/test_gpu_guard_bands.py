"""Output integrity on the GPU: guard bands around every buffer a kernel
writes, and caller ids outside [0,E).

compute-sanitizer is not used here; instead every output, and the workspace,
is carved out of a larger allocation whose bytes before and after it are
filled with a known pattern.  After each entry point has run, the bands
must be unchanged: no kernel writes past the buffers it was given.  The
entry points run on shapes that reach every kernel form (prefill with the
fp32-reduction and the fixed-order combine, CTA pairs, the decode path, the
four-call chain, the permutation without a workspace, the router and the
Gemma 4 block).
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_ffn_06_b200 import inputs
from parity_util import to_device

pytestmark = pytest.mark.gpu

BAND = 4096      # bytes on each side of a buffer (keeps 256-byte alignment)
PATTERN = 0xA5   # a NaN pattern in neither bf16 nor fp32, and no valid index


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixture_experts_ffn_06_b200 import api as a
    return a


class Guarded:
    """A buffer of ``shape`` and ``dtype`` inside an allocation whose BAND
    bytes on either side hold PATTERN."""

    def __init__(self, shape, dtype, fill=None):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.n = n
        self.raw = torch.full((BAND + n + BAND,), PATTERN, dtype=torch.uint8,
                              device="cuda")
        self.t = self.raw[BAND:BAND + n].view(dtype).view(*shape)
        if fill is not None:
            self.t.fill_(fill)

    def intact(self) -> bool:
        torch.cuda.synchronize()
        return bool((self.raw[:BAND] == PATTERN).all()) and \
            bool((self.raw[BAND + self.n:] == PATTERN).all())


def _ws(api, s):
    g = Guarded((api.moe_workspace_size(s),), torch.uint8)
    g.t[:256].zero_()
    return g


def _check_all(*bufs):
    for name, g in bufs:
        assert g.intact(), f"{name}: a guard band was overwritten"


SHAPES = {
    "ragged": (inputs.Shape(T=37, H=200, E=5, k=3, I=104, act=1), "uniform"),
    "shared": (inputs.Shape(T=40, H=128, E=6, k=2, I=96, n_shared=2,
                            I_shared=96), "ones"),
    "gemma_T130": (inputs.Shape(T=130, H=2816, E=128, k=8, I=704, act=1),
                   "uniform"),
    "pairs": (inputs.Shape(T=700, H=200, E=3, k=2, I=104, act=1), "uniform"),
    "few": (inputs.Shape(T=3, H=200, E=5, k=3, I=104, act=1), "uniform"),
}
VARIANTS = {"prefill": (1, False, 0), "prefill_det": (1, True, 0),
            "pairs": (1, False, 2), "decode": (2, False, 0)}


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("name", list(SHAPES))
def test_forward_writes_only_its_buffers(api, name, variant):
    shp, sc = SHAPES[name]
    inp = to_device(inputs.make_inputs(shp, seed=2, scale=sc))
    s = api.shape_from(shp)
    T, H, k = shp.T, shp.H, shp.k
    out = Guarded((T, H), torch.bfloat16)
    out32 = Guarded((T, H), torch.float32)
    ids = Guarded((T, k), torch.int32)
    w = Guarded((T, k), torch.float32)
    ws = _ws(api, s)
    path, det, pairs = VARIANTS[variant]
    for _ in range(2):  # the second call finds the first call's workspace
        api.moe_forward_ex(s, inp.x, inp.logits, inp.w13, inp.w2, inp.scale,
                           inp.w13_sh, inp.w2_sh, out.t, ws.t, ids_out=ids.t,
                           w_out=w.t, out_f32=out32.t, path=path,
                           deterministic=det, cta_pairs=pairs)
    assert api.moe_read_error(ws.t) == 0
    assert torch.isfinite(out32.t).all()
    _check_all(("out", out), ("out_f32", out32), ("ids", ids), ("w", w),
               ("workspace", ws))


@pytest.mark.parametrize("name", ["ragged", "shared", "pairs"])
def test_four_call_chain_writes_only_its_buffers(api, name):
    shp, sc = SHAPES[name]
    inp = to_device(inputs.make_inputs(shp, seed=3, scale=sc))
    s = api.shape_from(shp)
    T, H, k, S, E = shp.T, shp.H, shp.k, shp.n_shared, shp.E
    cap = api.moe_layout_capacity(s)
    ids = Guarded((T, k), torch.int32)
    w = Guarded((T, k), torch.float32)
    offsets = Guarded((E + S + 1,), torch.int32)
    sorted_slots = Guarded((cap,), torch.int32)
    slot_row = Guarded((T, k + S), torch.int32)
    y_perm = Guarded((cap, H), torch.float32)
    out = Guarded((T, H), torch.bfloat16)
    ws = _ws(api, s)
    api.moe_route(s, inp.logits, inp.scale, ids.t, w.t)
    api.moe_permute(s, ids.t, offsets.t, sorted_slots.t, slot_row.t, ws.t)
    api.moe_expert_ffn(s, inp.x, offsets.t, sorted_slots.t, inp.w13, inp.w2,
                       inp.w13_sh, inp.w2_sh, y_perm.t, ws.t)
    api.moe_combine(s, y_perm.t, slot_row.t, w.t, out.t)
    assert api.moe_read_error(ws.t) == 0
    _check_all(("ids", ids), ("w", w), ("offsets", offsets),
               ("sorted_slots", sorted_slots), ("slot_row", slot_row),
               ("y_perm", y_perm), ("out", out), ("workspace", ws))


def test_noalloc_router_and_block_write_only_their_buffers(api):
    # the permutation without a workspace
    T, E, k = 3000, 64, 6
    gen = torch.Generator().manual_seed(4)
    z = inputs.router_logits(T, E, k, gen, "cpu")
    ids = torch.topk(z, k, dim=-1).indices.to(torch.int32).cuda()
    s = api.make_shape(T=T, H=64, E=E, k=k, I=64)
    cap = api.moe_layout_capacity(s)
    offsets = Guarded((E + 1,), torch.int32)
    sorted_slots = Guarded((cap,), torch.int32)
    slot_row = Guarded((T, k), torch.int32)
    api.moe_permute_noalloc(s, ids, offsets.t, sorted_slots.t, slot_row.t)
    _check_all(("offsets", offsets), ("sorted_slots", sorted_slots),
               ("slot_row", slot_row))

    # the router ahead of the routing
    T, H, E = 70, 256, 24
    g = torch.Generator(device="cuda").manual_seed(5)
    rx, rw, rs = inputs.router_inputs(T, H, E, g, "cuda")
    s = api.make_shape(T=T, H=H, E=E, k=2, I=64)
    logits = Guarded((T, E), torch.float32)
    api.moe_router_logits(s, rx, rw, rs, 1e-6, logits.t)
    assert torch.isfinite(logits.t).all()
    _check_all(("logits", logits))

    # the Gemma 4 block, decode- and prefill-sized
    for T in (5, 70):
        shp = inputs.Shape(T=T, H=256, E=8, k=2, I=64, act=1)
        moe = to_device(inputs.make_inputs(shp, seed=6, scale="uniform"))
        blk = inputs.gemma4_block_inputs(T, 256, 8, 96, seed=7, device="cuda")
        s = api.shape_from(shp)
        out = Guarded((T, 256), torch.bfloat16)
        out32 = Guarded((T, 256), torch.float32)
        ws = Guarded((api.moe_gemma4_workspace_size(s, 96),), torch.uint8, fill=0)
        api.moe_gemma4_block(s, blk.x, blk.norms, 1e-6, blk.mlp_w13, blk.mlp_w2,
                             blk.router_w, blk.router_scale, 1e-6, moe.w13,
                             moe.w2, moe.scale, out.t, ws.t, out_f32=out32.t)
        assert torch.isfinite(out32.t).all()
        _check_all(("block out", out), ("block out_f32", out32),
                   ("block workspace", ws))


# ------------------------------------------------ ids outside [0, E)

def _layout_of_valid(ids: np.ndarray, E: int, P: int = 128):
    """Counting sort of the slots whose id is in [0,E), by brute force: the
    layout moe_permute must give when the other slots are dropped."""
    T, k = ids.shape
    flat = ids.ravel()
    offsets, rows = [0], []
    for e in range(E):
        seg = [s for s in range(T * k) if flat[s] == e]
        padded = (len(seg) + P - 1) // P * P
        rows += seg + [-1] * (padded - len(seg))
        offsets.append(offsets[-1] + padded)
    slot_row = np.full((T, k), -1, np.int64)
    for r, sl in enumerate(rows):
        if sl >= 0:
            slot_row[sl // k, sl % k] = r
    return np.array(offsets), np.array(rows), slot_row


def test_ids_outside_the_experts_are_dropped_and_reported(api):
    T, E, k = 300, 16, 4
    gen = torch.Generator().manual_seed(8)
    z = inputs.router_logits(T, E, k, gen, "cpu")
    ids_np = torch.topk(z, k, dim=-1).indices.to(torch.int32).numpy().copy()
    bad = [(0, 0, -1), (7, 2, E), (150, 1, E + 1000), (299, 3, 2 ** 31 - 1),
           (100, 0, -(2 ** 31))]
    for t, j, v in bad:
        ids_np[t, j] = v
    want_off, want_rows, want_slot_row = _layout_of_valid(ids_np, E)
    ids = torch.from_numpy(ids_np).cuda()
    s = api.make_shape(T=T, H=64, E=E, k=k, I=64)
    cap = api.moe_layout_capacity(s)
    for use_ws in (True, False):
        offsets = Guarded((E + 1,), torch.int32)
        sorted_slots = Guarded((cap,), torch.int32)
        slot_row = Guarded((T, k), torch.int32)
        if use_ws:
            ws = _ws(api, s)
            api.moe_permute(s, ids, offsets.t, sorted_slots.t, slot_row.t, ws.t)
            assert api.moe_read_error(ws.t) == 1  # MOE_ERR_INVALID_ARG
            assert api.moe_read_error(ws.t) == 0  # cleared
            _check_all(("workspace", ws))
        else:
            api.moe_permute_noalloc(s, ids, offsets.t, sorted_slots.t, slot_row.t)
        _check_all(("offsets", offsets), ("sorted_slots", sorted_slots),
                   ("slot_row", slot_row))
        assert np.array_equal(offsets.t.cpu().numpy(), want_off)
        n = int(want_off[-1])
        got_rows = sorted_slots.t.cpu().numpy()
        assert np.array_equal(got_rows[:n], want_rows)
        assert (got_rows[n:] == -1).all()
        assert np.array_equal(slot_row.t.cpu().numpy(), want_slot_row)

    # moe_combine adds nothing for a slot without a row
    H = 64
    y_perm = torch.randn(cap, H, device="cuda")
    w = torch.rand(T, k, device="cuda")
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    sr = torch.from_numpy(want_slot_row.astype(np.int32)).cuda()
    api.moe_combine(s, y_perm, sr, w, out)
    torch.cuda.synchronize()
    acc = torch.zeros(T, H)
    yc, wc, src = y_perm.cpu(), w.cpu(), want_slot_row
    for j in range(k):
        valid = torch.from_numpy(src[:, j] >= 0)
        rows = torch.from_numpy(np.where(src[:, j] >= 0, src[:, j], 0))
        prod = wc[:, j:j + 1] * yc[rows]
        acc = acc + torch.where(valid[:, None], prod, torch.zeros_like(prod))
    assert torch.equal(out.cpu(), acc.to(torch.bfloat16))
