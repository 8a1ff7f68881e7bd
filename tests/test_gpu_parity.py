"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Bars: top-k ids, the permutation and the slot maps bit-exact; gate weights
within 1e-6 relative; the layer output within max|err| <= 2e-2 x RMS(oracle),
checked on the fp32 result before its final rounding, while the bf16 output
must be exactly the round-to-nearest-even of that fp32 result and lie within
2e-2 x RMS + 2^-8 |oracle| (rounding a heavy-tailed output to bf16 alone can
exceed 2e-2 x RMS, so the bare bound cannot be put on the bf16 tensor).  Small shapes are compared on every output
element; the full-size workloads on every routing decision and on a token
sample with one token from every 128-row (expert, m-tile) of the layout.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_ffn_06_b200 import inputs
from parity_util import (assert_out_close, assert_routing_exact, gpu_forward,
                         oracle_forward, to_device)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from mixture_experts_ffn_06_b200 import api as a
    return a


SMALL = {
    "tiny": (inputs.shape_of("tiny"), "zero", "ones"),
    "ragged": (inputs.Shape(T=37, H=200, E=5, k=3, I=104, act=1), "zero", "uniform"),
    "tail704": (inputs.Shape(T=50, H=256, E=16, k=4, I=704, act=1), "zero", "uniform"),
    "shared": (inputs.Shape(T=40, H=128, E=6, k=2, I=96, n_shared=2, I_shared=96),
               "zero", "ones"),
    "single_expert": (inputs.Shape(T=19, H=64, E=1, k=1, I=64), "zero", "uniform"),
    "k_equals_E": (inputs.Shape(T=33, H=64, E=4, k=4, I=32, act=1), "zero", "uniform"),
    "one_token": (inputs.Shape(T=1, H=128, E=8, k=2, I=128), "zero", "uniform"),
    # T <= 8 on the decode path: the ring form of the skinny kernels, with a
    # K tail in both products (H % 32, I % 32), a partial 16-row block of I
    # and a partial 64-row block of H, and shared experts
    "few_ragged": (inputs.Shape(T=3, H=200, E=5, k=3, I=104, act=1), "zero",
                   "uniform"),
    "few_shared": (inputs.Shape(T=8, H=136, E=6, k=2, I=88, n_shared=2,
                                I_shared=88), "zero", "ones"),
    "gemma_shapes_T130": (inputs.Shape(T=130, H=2816, E=128, k=8, I=704, act=1),
                          "zero", "uniform"),
    # I a multiple of 88 but not of 128: the w13 GEMM runs its 176-row
    # (88 gate + 88 up) B tiles, here with a K tail (H = 72)
    "narrow_w13": (inputs.Shape(T=90, H=72, E=3, k=2, I=264), "normal0.5",
                   "uniform"),
    "wide_tiles": (inputs.Shape(T=300, H=520, E=3, k=2, I=392), "normal0.5", "uniform"),
    # T*k >= 256*E: the grouped GEMMs run on CTA pairs (M = 256), with odd
    # m-tile counts per expert, K and N tails, and shared experts
    "pairs_ragged": (inputs.Shape(T=700, H=200, E=3, k=2, I=104, act=1),
                     "normal0.5", "uniform"),
    "pairs_shared": (inputs.Shape(T=600, H=128, E=4, k=2, I=96, n_shared=1,
                                  I_shared=96), "zero", "ones"),
    # I >= 1024 and two m-tiles per expert: the w2 GEMM picks CTA pairs by
    # itself (also in moe_expert_ffn)
    "pairs_wide_I": (inputs.Shape(T=600, H=128, E=2, k=2, I=1024), "zero",
                     "uniform"),
}


def _small(name, seed=0):
    shp, bias, scale = SMALL[name]
    return inputs.make_inputs(shp, seed=seed, bias=bias, scale=scale)


PATHS = {"prefill": 1, "decode": 2}
# (path, deterministic combine, cta_pairs) variants of moe_forward_ex
VARIANTS = {"prefill": (1, False, 0), "prefill_det": (1, True, 0),
            "prefill_pairs": (1, False, 2), "prefill_pairs_det": (1, True, 2),
            "decode": (2, False, 0)}


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_small_every_element(api, name, variant):
    inp = _small(name)
    want, ids_ref, w_ref = oracle_forward(inp)
    path, det, pairs = VARIANTS[variant]
    out, out32, ids, w = gpu_forward(api, to_device(inp), path=path,
                                     deterministic=det, cta_pairs=pairs)
    assert_routing_exact(ids, w, ids_ref, w_ref)
    assert_out_close(out32, want, f"{name} ({variant})", bf16=out)


@pytest.mark.parametrize("path", list(PATHS))
def test_all_tokens_on_one_expert(api, path):
    # one expert takes every token: a segment of several M tiles (prefill)
    # or several 64-token passes (decode); the other experts are empty
    shp = inputs.Shape(T=300, H=128, E=8, k=1, I=256)
    inp = inputs.make_inputs(shp, seed=1)
    inp.logits[:, 5] += 50.0
    want, ids_ref, w_ref = oracle_forward(inp)
    assert (ids_ref == 5).all()
    out, out32, ids, w = gpu_forward(api, to_device(inp), path=PATHS[path])
    assert_routing_exact(ids, w, ids_ref, w_ref)
    assert_out_close(out32, want, f"one hot expert ({path})", bf16=out)


def _layout_gpu(api, s, ids_dev, E, S):
    cap = api.moe_layout_capacity(s)
    T, k = ids_dev.shape
    offsets = torch.full((E + S + 1,), -7, dtype=torch.int32, device="cuda")
    sorted_slots = torch.full((cap,), -7, dtype=torch.int32, device="cuda")
    slot_row = torch.full((T, k + S), -7, dtype=torch.int32, device="cuda")
    ws = api.alloc_workspace(s)
    api.moe_permute(s, ids_dev, offsets, sorted_slots, slot_row, ws)
    torch.cuda.synchronize()
    return offsets.cpu().numpy(), sorted_slots.cpu().numpy(), slot_row.cpu().numpy()


@pytest.mark.parametrize("name", ["tiny", "ragged", "shared", "gemma_shapes_T130",
                                  "one_token", "k_equals_E"])
def test_permute_bit_exact(api, name):
    inp = _small(name)
    shp = inp.shape
    s = api.shape_from(shp)
    ids_ref, _ = oracle.route(inp.logits, shp.k, scale=inp.scale)
    got = _layout_gpu(api, s, torch.from_numpy(ids_ref).cuda(), shp.E, shp.n_shared)
    want = oracle.layout(ids_ref, shp.E, shp.n_shared, 128)
    for g, w_, what in zip(got, want, ("offsets", "sorted_slots", "slot_row")):
        assert (g == w_).all(), what


def test_permute_large_random_ids(api):
    # many layout blocks (T*k > 1024) and skewed counts
    T, E, k, S = 5000, 64, 6, 2
    gen = torch.Generator().manual_seed(3)
    z = inputs.router_logits(T, E, k, gen, "cpu",
                             bias=(-1.1 * torch.log(torch.arange(E) + 1.0)).float())
    ids_ref, _ = oracle.route(z, k)
    s = api.make_shape(T=T, H=64, E=E, k=k, I=64, n_shared=S, I_shared=64)
    got = _layout_gpu(api, s, torch.from_numpy(ids_ref).cuda(), E, S)
    want = oracle.layout(ids_ref, E, S, 128)
    for g, w_, what in zip(got, want, ("offsets", "sorted_slots", "slot_row")):
        assert (g == w_).all(), what


@pytest.mark.parametrize("name", ["tiny", "ragged", "shared", "tail704",
                                  "pairs_ragged", "pairs_shared", "pairs_wide_I"])
def test_four_call_chain_against_oracle_rows(api, name):
    """moe_route -> moe_permute -> moe_expert_ffn -> moe_combine."""
    inp = _small(name)
    shp = inp.shape
    d = to_device(inp)
    s = api.shape_from(shp)
    T, k, S, H = shp.T, shp.k, shp.n_shared, shp.H
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    api.moe_route(s, d.logits, d.scale, ids, w)
    cap = api.moe_layout_capacity(s)
    offsets = torch.empty(shp.E + S + 1, dtype=torch.int32, device="cuda")
    sorted_slots = torch.empty(cap, dtype=torch.int32, device="cuda")
    slot_row = torch.empty(T, k + S, dtype=torch.int32, device="cuda")
    ws = api.alloc_workspace(s)
    api.moe_permute(s, ids, offsets, sorted_slots, slot_row, ws)
    y_perm = torch.empty(cap, H, dtype=torch.float32, device="cuda")
    api.moe_expert_ffn(s, d.x, offsets, sorted_slots, d.w13, d.w2, d.w13_sh,
                       d.w2_sh, y_perm, ws)
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    api.moe_combine(s, y_perm, slot_row, w, out)
    torch.cuda.synchronize()
    assert api.moe_read_error(ws) == 0

    # unweighted expert rows against the oracle, every row in use
    used = int(offsets[-1])
    slots = sorted_slots[:used].cpu().numpy()
    rows = np.nonzero(slots >= 0)[0]
    sl = slots[rows]
    R = T * k
    routed = sl < R
    ids_np = ids.cpu().numpy().ravel()
    y = y_perm[:used].cpu().numpy().astype(np.float64)
    if routed.any():
        want = oracle.expert_rows(inp.x, inp.w13, inp.w2, sl[routed] // k,
                                  ids_np[sl[routed]], shp.act)
        rms = np.sqrt(np.mean(want ** 2))
        assert np.abs(y[rows[routed]] - want).max() <= 2e-2 * rms
    if S:
        q = sl[~routed] - R
        want = oracle.expert_rows(inp.x, inp.w13_sh, inp.w2_sh, q % T, q // T,
                                  shp.act)
        rms = np.sqrt(np.mean(want ** 2))
        assert np.abs(y[rows[~routed]] - want).max() <= 2e-2 * rms
    pad = np.nonzero(slots < 0)[0]
    assert (y[pad] == 0).all()  # padding rows hold zeros

    # combine: the fixed-order fp32 sum of the rows it was given (each
    # product rounded to fp32, then added, j = 0..k-1, then the shared
    # experts), rounded once -- redone here op by op, so bit for bit
    sr = slot_row.long().cpu()
    yt = y_perm.cpu()
    acc = torch.zeros(T, H, dtype=torch.float32)
    wt = w.cpu()
    for j in range(k):
        prod = wt[:, j:j + 1] * yt[sr[:, j]]
        acc = acc + prod
    for sh in range(S):
        acc = acc + yt[sr[:, k + sh]]
    assert torch.equal(out.cpu(), acc.to(torch.bfloat16))

    # the chain's fp32 sum and the fused call both meet the output bound, and
    # the two paths use the same arithmetic: bit-identical outputs
    want, _, _ = oracle_forward(inp)
    assert_out_close(acc, want, name + " chain")
    fused, out32, _, _ = gpu_forward(api, d, path=PATHS["prefill"],
                                     deterministic=True)
    assert_out_close(out32, want, name + " fused", bf16=fused)
    assert torch.equal(out, fused)  # same GEMM kernels, same additions
    fast, fast32, _, _ = gpu_forward(api, d, path=PATHS["prefill"])
    assert_out_close(fast32, want, name + " fused, fp32 reductions")


@pytest.mark.parametrize("variant", ["prefill_det", "prefill_pairs_det", "decode"])
def test_repeat_calls_are_bit_identical(api, variant):
    inp = to_device(_small("gemma_shapes_T130"))
    path, det, pairs = VARIANTS[variant]
    a, a32, _, _ = gpu_forward(api, inp, path=path, deterministic=det,
                               cta_pairs=pairs)
    b, b32, _, _ = gpu_forward(api, inp, path=path, deterministic=det,
                               cta_pairs=pairs)
    assert torch.equal(a, b) and torch.equal(a32, b32)


@pytest.mark.parametrize("variant", ["prefill_det", "prefill_pairs_det", "decode"])
@pytest.mark.parametrize("name", ["ragged", "shared", "gemma_shapes_T130",
                                  "few_ragged"])
def test_stale_workspace_changes_nothing(api, name, variant):
    # Padding rows of the gathered activations and of h are never written;
    # each MMA row depends on its own A row only, so whatever they hold may
    # reach only padding rows of the products.  0xFF bytes are NaN in both
    # bf16 and fp32: one leaking into a real output would show.
    inp = to_device(_small(name))
    path, det, pairs = VARIANTS[variant]
    a, a32, _, _ = gpu_forward(api, inp, path=path, deterministic=det,
                               cta_pairs=pairs)
    b, b32, _, _ = gpu_forward(api, inp, path=path, deterministic=det,
                               cta_pairs=pairs, ws_fill=0xFF)
    assert torch.isfinite(b32).all()
    assert torch.equal(a, b) and torch.equal(a32, b32)


@pytest.mark.parametrize("path", list(PATHS))
def test_stage_events_may_be_left_out(api, path):
    # only the first and the last event: the step's time with no event
    # between its kernels
    inp = to_device(_small("gemma_shapes_T130" if path != "decode" else "one_token"))
    want, _, _, _ = gpu_forward(api, inp, path=PATHS[path])
    s = api.shape_from(inp.shape)
    out = torch.empty_like(want)
    ws = api.alloc_workspace(s)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    events = [ev[0]] + [None] * (api.NUM_STAGES - 1) + [ev[1]]
    api.moe_forward_ex(s, inp.x, inp.logits, inp.w13, inp.w2, inp.scale,
                       inp.w13_sh, inp.w2_sh, out, ws, events=events,
                       path=PATHS[path])
    torch.cuda.synchronize()
    assert api.moe_read_error(ws) == 0
    assert ev[0].elapsed_time(ev[1]) > 0
    if path == "decode":
        assert torch.equal(out, want)  # the decode path is deterministic
    else:  # fp32 reductions in any order, then one bf16 rounding
        assert (out.float() - want.float()).abs().max() <= \
            1e-2 * want.float().abs().max()


def test_fast_combine_repeats_within_fp32_rounding(api):
    inp = to_device(_small("gemma_shapes_T130"))
    _, a32, _, _ = gpu_forward(api, inp, path=PATHS["prefill"])
    _, b32, _, _ = gpu_forward(api, inp, path=PATHS["prefill"])
    # k + S <= 9 fp32 terms per element, added in any order
    assert (a32 - b32).abs().max().item() <= 1e-5 * a32.abs().max().item()


def test_device_wait_limit_reports_timeout(api):
    s = api.make_shape(T=8, H=64, E=4, k=2, I=64)
    ws = api.alloc_workspace(s)
    api.moe_selftest_wait_timeout(ws, 2000)
    assert api.moe_read_error(ws) == 5  # MOE_ERR_TIMEOUT, context still usable
    assert api.moe_read_error(ws) == 0  # cleared
    inp = to_device(inputs.make_inputs(inputs.Shape(T=8, H=64, E=4, k=2, I=64)))
    out, _, _, _ = gpu_forward(api, inp)
    assert torch.isfinite(out.float()).all()


def test_workspace_too_small_is_refused(api):
    inp = to_device(_small("tiny"))
    s = api.shape_from(inp.shape)
    ws = torch.zeros(api.moe_workspace_size(s) - 256, dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(inp.shape.T, inp.shape.H, dtype=torch.bfloat16,
                      device="cuda")
    with pytest.raises(api.MoEError) as e:
        api.moe_forward(s, inp.x, inp.logits, inp.w13, inp.w2, inp.scale,
                        None, None, out, ws)
    assert e.value.status == 3


# ----------------------------------------------------------- full workloads

@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name", ["decode_t1", "decode_t4", "decode_t16",
                                  "decode_t64", "decode_t256"])
def test_decode_sweep_every_element(api, name, path):
    inp = inputs.make_inputs(name, seed=0, device="cuda")
    out, out32, ids, w = gpu_forward(api, inp, path=PATHS[path])
    want, ids_ref, w_ref = oracle_forward(inp)
    assert_routing_exact(ids, w, ids_ref, w_ref)
    assert_out_close(out32, want, name, bf16=out)


def _tile_tokens(offsets, sorted_slots, T, k, seed, P=128):
    """One token from every P-row (expert, m-tile) of the layout, shared
    experts' segments included: a seeded pick among the tile's real rows
    (the last tile of a segment holds padding rows as well), plus the first
    and last token.  Every tile of both grouped GEMMs then has at least one
    of its rows compared with the oracle."""
    rng = np.random.default_rng(seed)
    R = T * k
    chosen = {0, T - 1}
    n_tiles = 0
    for g in range(len(offsets) - 1):
        for r0 in range(int(offsets[g]), int(offsets[g + 1]), P):
            rows = sorted_slots[r0:r0 + P]
            real = rows[rows >= 0]
            if real.size == 0:
                continue
            n_tiles += 1
            s = int(real[rng.integers(real.size)])
            chosen.add(s // k if s < R else (s - R) % T)
    return np.array(sorted(chosen), np.int64), n_tiles


_FULL_CACHE = {}


def _full_case(name):
    """Inputs on the device, and the oracle's routing, layout and the output
    of the tile-covering token sample (computed once per workload)."""
    inp = inputs.make_inputs(name, seed=0, device="cuda")
    if name not in _FULL_CACHE:
        shp = inp.shape
        ids_ref, w_ref = oracle.route(inp.logits, shp.k, scale=inp.scale)
        lay = oracle.layout(ids_ref, shp.E, shp.n_shared, 128)
        tok, n_tiles = _tile_tokens(lay[0], lay[1], shp.T, shp.k, seed=1)
        want_out, _, _ = oracle_forward(inp, tokens=tok)
        _FULL_CACHE[name] = (ids_ref, w_ref, lay, tok, n_tiles, want_out)
    return (inp,) + _FULL_CACHE[name]


# Tokens compared per workload (one per tile): Mixtral ~70 of 4096,
# many-small ~560 of 8192, skewed ~1030 of 16384.
@pytest.mark.parametrize("det,pairs", [(False, 0), (True, 0), (False, 2)])
@pytest.mark.parametrize("name", ["mixtral_prefill", "many_small_prefill",
                                  "skewed_shared_prefill"])
def test_prefill_full_size(api, name, det, pairs):
    inp, ids_ref, w_ref, want_lay, tok, n_tiles, want_out = _full_case(name)
    shp = inp.shape
    out, out32, ids, w = gpu_forward(api, inp, deterministic=det,
                                     cta_pairs=pairs)
    # routing of every token, bit-exact ids
    assert_routing_exact(ids, w, ids_ref, w_ref)
    # permutation of every slot
    s = api.shape_from(shp)
    got = _layout_gpu(api, s, ids, shp.E, shp.n_shared)
    for g, w_, what in zip(got, want_lay, ("offsets", "sorted_slots", "slot_row")):
        assert (g == w_).all(), what
    # outputs of one token from every (expert, m-tile)
    assert len(tok) >= n_tiles // shp.k, (len(tok), n_tiles)
    sel = torch.from_numpy(tok).cuda()
    assert_out_close(out32[sel], want_out, f"{name}: {len(tok)} tokens, "
                     f"{n_tiles} tiles", bf16=out[sel])


@pytest.mark.parametrize("E,k", [(5, 3), (128, 8), (64, 6), (512, 32), (40, 32)])
def test_route_ties_and_signed_zeros(api, E, k):
    # Logits drawn from a handful of values, so that most rows hold exact ties
    # (-0.0 and +0.0 among them, which compare equal): the ids must follow
    # (larger logit, then lower id) and the weights the oracle's.
    gen = torch.Generator().manual_seed(E * 100 + k)
    T = 300
    vals = torch.tensor([-1.5, -0.0, 0.0, 0.25, 0.25, 2.0, -3.0],
                        dtype=torch.float32)
    z = vals[torch.randint(0, len(vals), (T, E), generator=gen)]
    z[0] = 0.0
    z[1] = -0.0
    z[2, ::2] = -0.0
    z[2, 1::2] = 0.0
    s = api.make_shape(T=T, H=64, E=E, k=k, I=64)
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    api.moe_route(s, z.cuda(), None, ids, w)
    torch.cuda.synchronize()
    ids_ref, w_ref = oracle.route(z.numpy(), k)
    assert (ids.cpu().numpy() == ids_ref).all()
    np.testing.assert_allclose(w.cpu().numpy(), w_ref, rtol=1e-6, atol=0)
