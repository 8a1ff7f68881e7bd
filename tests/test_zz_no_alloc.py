"""moe_permute_noalloc: the permutation for callers that cannot allocate.

Callers that run inside a CUDA graph capture, or whose runtime forbids
device allocations at launch time, cannot hand the library a workspace.
moe_permute_noalloc keeps its scratch in a fixed device array inside the
library instead.  These tests check that it returns exactly what the
workspace-based moe_permute returns, on two calls in a row (the second call
finds the first call's leftovers in the shared array), and that batches
beyond its fixed limit are refused before anything runs.

This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_ffn_06_b200 import inputs


@pytest.fixture(scope="module")
def api():
    from mixture_experts_ffn_06_b200 import build
    build.build()
    from mixture_experts_ffn_06_b200 import api as a
    return a


def _ids(T, E, k, seed, zipf=False):
    gen = torch.Generator().manual_seed(seed)
    bias = (-1.1 * torch.log(torch.arange(E) + 1.0)).float() if zipf else None
    z = inputs.router_logits(T, E, k, gen, "cpu", bias=bias)
    return torch.topk(z, k, dim=-1).indices.to(torch.int32)


def _outputs(api, s, E, S, T, k):
    cap = api.moe_layout_capacity(s)
    return (torch.full((E + S + 1,), -7, dtype=torch.int32, device="cuda"),
            torch.full((cap,), -7, dtype=torch.int32, device="cuda"),
            torch.full((T, k + S), -7, dtype=torch.int32, device="cuda"))


@pytest.mark.gpu
def test_noalloc_matches_workspace_permute_twice_in_a_row(api):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # the second case is smaller, so the first call's scratch is still there
    cases = [(16000, 64, 6, 2, True), (700, 128, 8, 0, False)]
    for call, (T, E, k, S, zipf) in enumerate(cases):
        ids = _ids(T, E, k, seed=call, zipf=zipf).cuda()
        s = api.make_shape(T=T, H=64, E=E, k=k, I=64, n_shared=S,
                           I_shared=64 if S else 0)
        ref = _outputs(api, s, E, S, T, k)
        ws = api.alloc_workspace(s)
        api.moe_permute(s, ids, *ref, ws)
        got = _outputs(api, s, E, S, T, k)
        api.moe_permute_noalloc(s, ids, *got)
        torch.cuda.synchronize()
        for r, g, what in zip(ref, got, ("offsets", "sorted_slots", "slot_row")):
            assert torch.equal(r, g), f"call {call}: {what} differs"
        # the permutation itself is sane: every slot appears exactly once
        used = int(got[0][-1])
        slots = got[1][:used].cpu().numpy()
        assert np.array_equal(np.sort(slots[slots >= 0]),
                              np.arange(T * (k + S)))


def test_noalloc_refuses_batches_over_its_limit(api):
    # rejected on the host before any CUDA call, so no GPU is needed
    limit = 131072  # MOE_NOALLOC_MAX_SLOTS
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced
    over = api.make_shape(T=limit // 8 + 1, H=64, E=128, k=8, I=64)
    rc = api.lib.moe_permute_noalloc(ctypes.byref(over), fake, fake, fake,
                                     fake, null)
    assert rc == 2  # MOE_ERR_UNSUPPORTED
    bad = api.make_shape(T=10, H=64, E=4, k=5, I=64)  # k > E
    rc = api.lib.moe_permute_noalloc(ctypes.byref(bad), fake, fake, fake,
                                     fake, null)
    assert rc == 1  # MOE_ERR_INVALID_ARG


def _distinct_ids(T, E, k, seed):
    # k distinct experts per token, uniformly random (no margin needed: the
    # permutation takes ids, not logits)
    g = torch.Generator().manual_seed(seed)
    return torch.rand(T, E, generator=g).argsort(dim=1)[:, :k].to(torch.int32)


@pytest.mark.gpu
def test_noalloc_at_its_limit_with_512_experts(api):
    # T*k == MOE_NOALLOC_MAX_SLOTS and E = 512: every layout block's counts
    # use the full 512-expert stride of the scratch, and layout_count needs
    # its shared-memory opt-in (32 warps x 512 counters)
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    T, E, k = 16384, 512, 8
    assert T * k == 131072
    ids = _distinct_ids(T, E, k, seed=11).cuda()
    s = api.make_shape(T=T, H=64, E=E, k=k, I=64)
    ref = _outputs(api, s, E, 0, T, k)
    ws = api.alloc_workspace(s)
    api.moe_permute(s, ids, *ref, ws)
    got = _outputs(api, s, E, 0, T, k)
    api.moe_permute_noalloc(s, ids, *got)
    torch.cuda.synchronize()
    for r, g, what in zip(ref, got, ("offsets", "sorted_slots", "slot_row")):
        assert torch.equal(r, g), what


@pytest.mark.gpu
def test_noalloc_call_captured_in_a_cuda_graph(api):
    # the use case of the entry point: one call before capture (it looks up
    # the scratch address), then a call recorded into a CUDA graph and
    # replayed, with new ids copied into the captured input buffer
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    T, E, k = 5000, 128, 8
    s = api.make_shape(T=T, H=64, E=E, k=k, I=64)
    ids = _distinct_ids(T, E, k, seed=12).cuda()
    outs = _outputs(api, s, E, 0, T, k)
    api.moe_permute_noalloc(s, ids, *outs)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        api.moe_permute_noalloc(s, ids, *outs, stream=stream)
    for seed in (13, 14):
        ids.copy_(_distinct_ids(T, E, k, seed=seed).cuda())
        graph.replay()
        torch.cuda.synchronize()
        ref = _outputs(api, s, E, 0, T, k)
        ws = api.alloc_workspace(s)
        api.moe_permute(s, ids, *ref, ws)
        torch.cuda.synchronize()
        for r, g, what in zip(ref, outs, ("offsets", "sorted_slots", "slot_row")):
            assert torch.equal(r, g), f"replay {seed}: {what}"
    del graph
