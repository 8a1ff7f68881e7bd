"""Benchmark of the sparse MoE feed-forward layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config mixtral_prefill]

One step is one whole layer (route, permute, expert FFN, combine) over one
batch of synthetic tokens, through the C ABI call ``moe_forward``.  The
default workload is the Mixtral-shaped prefill (T=4096, H=4096, E=8, k=2,
I=14336, SiLU).  Inputs are resident in HBM when the timed region starts; the
expert weights (2.8 GB) are far larger than L2, so every step streams them
from HBM.  A small batch that touches few experts (weights under four times
the L2 size) gets an L2 flush before every step, outside that step's CUDA
events.  ``e2e`` repeats the measurement with the token inputs copied from
pinned host memory and the output copied back inside the timed region.

With N > 1 (torchrun, one rank per GPU) every rank runs its own replica of
the layer on its own batch: the layer has no cross-GPU exchange, so there is
no collective on the data path (weak scaling).

The default run (the Mixtral-shaped headline, one GPU) adds a ``configs``
key with one entry for each other workload of the benchmark -- the
many-small-experts and skewed prefills, the decode sweep T = 1, 4, 16, 64,
256, and the Mixtral-shaped and many-small prefills and decode T = 4, 16,
64 with FP8 (e4m3) experts -- each device-timed the same way, with its roofline fraction, its
CPU baseline and ``parity``: the layer outputs the oracle computed for the
baseline's token sample set beside the GPU's (max |err| / RMS of the fp32
and bf16 outputs), and the routing ids, gate weights and layout of the whole
batch compared with the oracle's.  The headline carries the same ``parity``.
``--headline-only`` leaves the other workloads out; ``--fp8`` runs the
headline with FP8 experts (``moe_forward_fp8``, prefill path).

``--impl reference`` times the fp64 CPU oracle on the host cores instead (a
bounded token sample per step) and prints the same line with
``"impl": "reference"``.

``--block I_DENSE`` times the Gemma 4 MoE block instead (the config's MoE
with a parallel dense MLP of that intermediate size, the router on the
residual and the five gamma norms; one GPU, device-timed).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import select
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("MoE layer tokens/s on 1 B200 + % of roofline "
          "(bf16 TFLOPS prefill / HBM GB/s decode)")
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", default="mixtral_prefill")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--shape", default=None,
                    help="override the workload shape, e.g. T=4096,I=2048")
    ap.add_argument("--path", choices=("auto", "prefill", "decode"),
                    default="auto", help="force the kernel path")
    ap.add_argument("--deterministic", action="store_true",
                    help="fixed-order combine on the prefill path")
    ap.add_argument("--pairs", choices=("auto", "off", "on"), default="auto",
                    help="prefill GEMMs on single CTAs or on CTA pairs")
    ap.add_argument("--no-graph", action="store_true",
                    help="time plain stream launches instead of one CUDA graph")
    ap.add_argument("--profile", action="store_true",
                    help="device timing only: skip the e2e and CPU legs")
    ap.add_argument("--block", type=int, default=0, metavar="I_DENSE",
                    help="time the Gemma 4 MoE block (dense MLP of this "
                         "intermediate size in parallel with the MoE, gamma "
                         "norms, router on the residual) instead of the layer")
    ap.add_argument("--fp8", action="store_true",
                    help="FP8 experts (e4m3 weights with per-row scales, moe_forward_fp8)")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the other workloads' lines (the configs key)")
    ap.add_argument("--router", action="store_true",
                    help="start from hidden states: the router (RMSNorm, scale, "
                         "GateLinear) computes the logits inside every step")
    return ap.parse_args()


def make_workload(args, device, seed):
    from mixture_experts_ffn_06_b200 import inputs
    over = {}
    if args.shape:
        for kv in args.shape.split(","):
            key, val = kv.split("=")
            over[key.strip()] = int(val)
    return inputs.make_inputs(args.config, seed=seed, device=device, **over)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def workload_name(cfg_name, shp):
    act = "SiLU" if shp.act == 0 else "tanh-GELU"
    s = (f"{cfg_name}: T={shp.T} H={shp.H} E={shp.E} k={shp.k} I={shp.I} "
         f"{act}")
    if shp.n_shared:
        s += f" + {shp.n_shared} shared (I={shp.I_shared})"
    return s


def max_over_ranks_fn(world: int, device):
    """The slowest rank's value of a per-rank time (all-reduce MAX); every
    rank takes the same collective step."""
    import torch
    import torch.distributed as dist

    def max_over_ranks(v: float) -> float:
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return max_over_ranks


def whole_job_rate(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Tokens/s of the whole job: every replica processes its own batch of
    tokens_per_rank tokens per step, and the step takes the slowest rank's
    time."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                "bf16_tflops_sustained": 1400.0}, "fallback"


_NVML_POLL = r"""
import sys, time
import pynvml
pynvml.nvmlInit()
try:
    h = pynvml.nvmlDeviceGetHandleByUUID(sys.argv[1])
except Exception:
    h = pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[2]))
reasons = (getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
           or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons)
print("max", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
while True:
    print(time.monotonic(), pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
          reasons(h), flush=True)
    time.sleep(0.001)
"""


class ClockSampler:
    """SM clock and throttle-reason sampling while the timed region runs.
    A child process polls NVML every millisecond and stamps each sample
    with the monotonic clock (the device found by its UUID, so that a
    CUDA_VISIBLE_DEVICES mapping is followed); the caller marks the timed
    region (begin / end) and only the samples inside it are reported (at
    least the first one after its start).  Without NVML, nvidia-smi every
    100 ms.  Reads only; changes no setting."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,"
             "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (hw_slowdown with the power brake)
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8 | 0x80,
                   "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self._t = None
        self.nvml = False
        self.sm_max = None
        self.t_begin = self.t_end = None

    def _uuid(self):
        try:
            import torch
            u = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            return ""

    def start(self):
        try:
            self.proc = subprocess.Popen(
                [sys.executable, "-c", _NVML_POLL, self._uuid(), str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            # the child is sampling once it has printed the maximum clock
            # (bounded wait: a child stuck in NVML falls back to nvidia-smi)
            ready, _, _ = select.select([self.proc.stdout], [], [], 10.0)
            first = self.proc.stdout.readline().split() if ready else []
            if len(first) == 2 and first[0] == "max":
                self.sm_max = float(first[1])
                self.nvml = True
            else:
                self._kill()
        except (OSError, ValueError):
            self._kill()
        if not self.nvml:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None
                return
            time.sleep(0.3)  # let nvidia-smi start
        self._t = threading.Thread(target=self._read, daemon=True)
        self._t.start()

    def begin(self):
        self.t_begin = time.monotonic()

    def end(self):
        self.t_end = time.monotonic()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def _kill(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()

    def _stamp(self, ln):
        try:
            return float(ln.split()[0])
        except (ValueError, IndexError):
            return None

    def stop(self):
        if self.proc is None:
            return None
        if self.nvml and self.t_begin is not None:
            # a timed region shorter than a sampling period: wait (briefly)
            # for the first sample taken after its start
            deadline = time.monotonic() + 0.2
            while time.monotonic() < deadline and not any(
                    (self._stamp(ln) or 0.0) >= self.t_begin for ln in self.lines[-4:]):
                time.sleep(0.002)
        self._kill()
        if self._t:
            self._t.join(timeout=5)
        if self.nvml:
            rows = []
            for ln in self.lines:
                parts = ln.split()
                try:
                    rows.append((float(parts[0]), float(parts[1]), int(parts[2])))
                except (ValueError, IndexError):
                    continue
            b = self.t_begin if self.t_begin is not None else float("-inf")
            e = self.t_end if self.t_end is not None else float("inf")
            inside = [r for r in rows if b <= r[0] <= e]
            if not inside:
                inside = [r for r in rows if r[0] >= b][:1]
            if not inside:
                return None
            bits = 0
            for r in inside:
                bits |= r[2]
            return {"sm_mhz": statistics.median(r[1] for r in inside),
                    "sm_max_mhz": self.sm_max,
                    "reasons": sorted(n for n, m in self.REASON_BITS.items() if bits & m),
                    "samples": len(inside),
                    "source": "nvml every 1 ms, samples inside the timed region"}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvidia-smi every 100 ms"}


def traffic_for(kernel_src: str, config: str, shape_override):
    """DRAM bytes per launch from the committed ncu summary, only for the
    workload it was captured on and while the kernel source still matches
    the one the counters were taken on."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    src = os.path.join(ROOT, "mixture_experts_ffn_06_b200", "csrc", kernel_src)
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    ent = d.get(kernel_src)
    if not ent or ent.get("source_sha256_16") != sha:
        return None
    if shape_override or ent.get("config") != config:
        return None
    return ent.get("bytes_per_launch")


# ----------------------------------------------------------- CPU baseline

def cpu_baseline_leg(inp, gpu, budget_s: float, max_rounds: int = 64, seed: int = 1,
                     fp8=None):
    """The CPU baseline: the oracle as it stands, timed on the host cores, on
    rounds of ``cores`` tokens drawn from the batch until ``budget_s`` has
    passed.  The layer outputs it computes for those tokens are then set
    beside the GPU's for the same tokens, and the routing and the layout of
    the whole batch beside the library's (``gpu``: host copies of one call's
    out, out_f32, ids, w and moe_permute's offsets / sorted_slots /
    slot_row).  Returns (baseline, parity) dicts."""
    import numpy as np
    import oracle
    cores = oracle.num_threads()
    shp = inp.shape
    T = shp.T
    host = {k: (None if v is None else v.cpu()) for k, v in
            dict(x=inp.x, logits=inp.logits, w13=inp.w13, w2=inp.w2,
                 scale=inp.scale, w13_sh=inp.w13_sh, w2_sh=inp.w2_sh).items()}
    xu = oracle._u16(host["x"])
    if fp8 is None:
        w13u, w2u = oracle._u16(host["w13"]), oracle._u16(host["w2"])
        sh13, sh2 = oracle._u16(host["w13_sh"]), oracle._u16(host["w2_sh"])
    else:  # FP8Experts on the device: codes and scales on the host
        t = fp8
        cv = lambda a: None if a is None else a.cpu()  # noqa: E731
        fp8 = (cv(t.w13_q), cv(t.w13_s), cv(t.w2_q), cv(t.w2_s))
        fp8_sh = (cv(t.sh13_q), cv(t.sh13_s), cv(t.sh2_q), cv(t.sh2_s))
    rng = np.random.default_rng(seed)
    per_round = min(cores, T)
    done, elapsed, rounds = 0, 0.0, 0
    toks, outs, slacks = [], [], []
    while rounds < max_rounds and (elapsed < budget_s or rounds == 0):
        tok = np.sort(rng.choice(T, per_round, replace=False))
        t0 = time.perf_counter()
        if fp8 is None:
            o, _, _ = oracle.forward(xu, host["logits"], w13u, w2u, shp.k, shp.act,
                                     scale=host["scale"], w13_sh=sh13, w2_sh=sh2,
                                     tokens=tok, nthreads=per_round)
        else:
            # with the validity slack of the intermediate's quantisation
            o, _, _, sl = oracle.forward_fp8(xu, host["logits"], *fp8, shp.k, shp.act,
                                             scale=host["scale"], sh13_q=fp8_sh[0],
                                             sh13_s=fp8_sh[1], sh2_q=fp8_sh[2],
                                             sh2_s=fp8_sh[3], tokens=tok,
                                             nthreads=per_round, with_slack=True)
            slacks.append(sl)
        elapsed += time.perf_counter() - t0
        toks.append(tok)
        outs.append(o)
        done += per_round
        rounds += 1
    baseline = {"value": done / elapsed, "unit": UNIT, "cores": per_round,
                "kind": "oracle",
                "sample": f"{done} tokens drawn from the same {T}-token batch in "
                          f"rounds of {per_round}, full layer per token (fp64"
                          f"{', FP8 experts' if fp8 is not None else ''}), "
                          f"{elapsed:.1f} s"}

    tok = np.concatenate(toks)
    want = np.concatenate(outs)
    slack = np.concatenate(slacks) if slacks else 0.0
    got32 = gpu["out_f32"][tok].astype(np.float64)
    gotbf = gpu["out"][tok].astype(np.float64)
    rms = float(np.sqrt(np.mean(want ** 2)))
    bound = 2e-2 * rms + 2.0 ** -8 * np.abs(want) + slack
    ids_ref, w_ref = oracle.route(host["logits"], shp.k, scale=host["scale"])
    lay = oracle.layout(ids_ref, shp.E, shp.n_shared, 128)
    lay_bad = sum(int((np.asarray(g) != np.asarray(w)).sum())
                  for g, w in zip(gpu["layout"], lay))
    parity = {
        "tokens_compared": int(np.unique(tok).size),
        "out_f32_max_err_over_rms": float(np.abs(got32 - want).max() / rms),
        "out_bf16_max_err_over_rms": float(np.abs(gotbf - want).max() / rms),
        "bf16_within_bound": bool((np.abs(gotbf - want) <= bound).all()),
        "ids_mismatched": int((gpu["ids"] != ids_ref).sum()),
        "weights_max_rel_err": float((np.abs(gpu["w"].astype(np.float64) - w_ref)
                                      / np.abs(w_ref)).max()),
        "layout_entries_mismatched": lay_bad,
        "tolerance": "out_f32 max|err| <= 2e-2 x RMS(oracle); bf16 within "
                     "2e-2 x RMS + 2^-8 |oracle|; ids and layout bit-exact; "
                     "weights 1e-6 relative"
                     + ("; FP8: both output bounds + the oracle's validity slack "
                        "of the intermediate's quantisation decisions"
                        if fp8 is not None else ""),
    }
    f32_ok = bool((np.abs(got32 - want) <= 2e-2 * rms + slack).all())
    if fp8 is not None:
        parity["out_f32_within_bound_with_slack"] = f32_ok
        parity["max_slack_over_rms"] = float(np.max(slack) / rms)
    parity["pass"] = (f32_ok
                      and parity["bf16_within_bound"]
                      and parity["ids_mismatched"] == 0
                      and parity["layout_entries_mismatched"] == 0
                      and parity["weights_max_rel_err"] <= 1e-6)
    return baseline, parity


# ---------------------------------------------------------------- our arm

def touched_experts(api, s, inp) -> int:
    """Distinct experts the batch routes to (+ shared experts), from one call
    of the library's own routing."""
    import torch
    shp = inp.shape
    ids = torch.empty(shp.T, shp.k, dtype=torch.int32, device=inp.x.device)
    w = torch.empty(shp.T, shp.k, dtype=torch.float32, device=inp.x.device)
    api.moe_route(s, inp.logits, inp.scale, ids, w)
    return int(torch.unique(ids).numel()) + shp.n_shared


def gpu_result(api, inp, s, path, args, fp8=None):
    """One call of the layer with every optional output, copied to the host
    (for the parity comparison of the CPU-baseline leg)."""
    import torch
    shp = inp.shape
    dev = inp.x.device
    ws = api.alloc_workspace_fp8(s, dev) if fp8 is not None else api.alloc_workspace(s, dev)
    out = torch.empty(shp.T, shp.H, dtype=torch.bfloat16, device=dev)
    out32 = torch.empty(shp.T, shp.H, dtype=torch.float32, device=dev)
    ids = torch.empty(shp.T, shp.k, dtype=torch.int32, device=dev)
    w = torch.empty(shp.T, shp.k, dtype=torch.float32, device=dev)
    pairs = {"auto": 0, "off": 1, "on": 2}[args.pairs]
    if fp8 is not None:
        api.moe_forward_fp8(s, inp.x, inp.logits, fp8_weights(api, fp8), inp.scale, out, ws,
                            ids_out=ids, w_out=w, out_f32=out32, path=path,
                            deterministic=args.deterministic, cta_pairs=pairs)
    else:
        api.moe_forward_ex(s, inp.x, inp.logits, inp.w13, inp.w2, inp.scale, inp.w13_sh,
                           inp.w2_sh, out, ws, ids_out=ids, w_out=w, out_f32=out32,
                           path=path, deterministic=args.deterministic, cta_pairs=pairs)
    cap = api.moe_layout_capacity(s)
    G = shp.E + shp.n_shared
    lay = (torch.empty(G + 1, dtype=torch.int32, device=dev),
           torch.empty(cap, dtype=torch.int32, device=dev),
           torch.empty(shp.T, shp.k + shp.n_shared, dtype=torch.int32, device=dev))
    api.moe_permute(s, ids, *lay, ws)
    torch.cuda.synchronize()
    if api.moe_read_error(ws) != 0:
        raise RuntimeError("device error in the parity call")
    return {"out": out.float().cpu().numpy(), "out_f32": out32.cpu().numpy(),
            "ids": ids.cpu().numpy(), "w": w.cpu().numpy(),
            "layout": tuple(t.cpu().numpy() for t in lay)}


def fp8_weights(api, fp):
    """moe_fp8_experts of an inputs.FP8Experts held on the device."""
    return api.fp8_experts(fp.w13_q, fp.w13_s, fp.w2_q, fp.w2_s, fp.sh13_q, fp.sh13_s,
                           fp.sh2_q, fp.sh2_s)


def timed_steps(args, api, inp, s, ws, out, stream, path, router, barrier,
                max_over_ranks, sample_clocks_gpu=None, fp8=None):
    """Device time of K steps of one workload.  By default the K steps are
    captured once into a CUDA graph and the timed region is one replay of
    it, so that host launch overhead does not pace small batches (the
    library makes no allocation or synchronisation, so its calls capture as
    they are); a second graph with an event between the stages gives the
    per-stage times.  A step whose expert weights (the distinct experts it
    routes to) fit a few times over in L2 would find them there on the next
    step: then every step is preceded by a write of twice the L2 size,
    outside that step's events, and the step time is the mean of the
    per-step event pairs; larger working sets stream from HBM by themselves.
    Returns a dict (ms_per_step, stage_ms, touched, weight_set, flush, ...)."""
    import torch
    shp = inp.shape
    dev = inp.x.device

    w8 = fp8_weights(api, fp8) if fp8 is not None else None

    def step(events=None):
        pairs = {"auto": 0, "off": 1, "on": 2}[args.pairs]
        if w8 is not None:
            api.moe_forward_fp8(s, inp.x, inp.logits if router is None else None, w8,
                                inp.scale, out, ws, events=events, path=path,
                                deterministic=args.deterministic, cta_pairs=pairs,
                                router=router)
            return
        api.moe_forward_ex(s, inp.x, inp.logits if router is None else None, inp.w13,
                           inp.w2, inp.scale, inp.w13_sh, inp.w2_sh, out, ws,
                           events=events, path=path, deterministic=args.deterministic,
                           cta_pairs=pairs, router=router)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    status = api.moe_read_error(ws)
    if status != 0:
        raise RuntimeError(f"device error during warm-up: {status}")

    touched = touched_experts(api, s, inp)
    weight_set = touched * 3.0 * shp.H * shp.I * (1 if fp8 is not None else 2)
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = None
    if weight_set < 4 * l2_bytes:
        flush_buf = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev)

    def flush(i):
        if flush_buf is not None:
            with torch.cuda.stream(stream):  # ordered before the step's kernels
                flush_buf.fill_(i & 0xFF)

    nst = api.NUM_STAGES
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)]
                for _ in range(args.steps)]
    # with the flush: only the first and last event of each step, so that no
    # event node sits between the step's kernels
    step_ev = [[e[0]] + [None] * (nst - 1) + [e[nst]] for e in
               [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)]
                for _ in range(args.steps)]]
    for evs in stage_ev + step_ev:  # create the events before the timed region
        for e in evs:
            if e is not None:
                e.record(stream)

    def plain_step(i):
        flush(i)
        step(step_ev[i] if flush_buf is not None else None)

    def staged_step(i):
        flush(i)
        step(stage_ev[i])

    graph = staged = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(args.steps):
                plain_step(i)
        staged = torch.cuda.CUDAGraph()
        with torch.cuda.graph(staged, stream=stream):
            for i in range(args.steps):
                staged_step(i)
        graph.replay()  # untimed first replays
        staged.replay()
        torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(sample_clocks_gpu) if sample_clocks_gpu is not None else None
    barrier()
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.start()
        clocks.begin()
    t_start.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for i in range(args.steps):
            plain_step(i)
    t_end.record(stream)
    if clocks is not None:
        torch.cuda.synchronize()
        clocks.end()  # the clock samples cover the timed steps only
    if staged is not None:
        staged.replay()
    else:
        for i in range(args.steps):
            staged_step(i)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop() if clocks is not None else None
    if graph is not None:
        del graph, staged
    if flush_buf is None:
        ms_total = t_start.elapsed_time(t_end)
    else:
        ms_total = sum(e[0].elapsed_time(e[nst]) for e in step_ev)
    ms_per_step = max_over_ranks(ms_total) / args.steps
    try:
        stage_ms = [statistics.mean(ev[j].elapsed_time(ev[j + 1])
                                    for ev in stage_ev) for j in range(nst)]
    except RuntimeError:
        # events inside the graph could not be timed: take the stage times
        # from the same K steps launched on the stream instead
        for i in range(args.steps):
            staged_step(i)
        torch.cuda.synchronize()
        stage_ms = [statistics.mean(ev[j].elapsed_time(ev[j + 1])
                                    for ev in stage_ev) for j in range(nst)]
    status = api.moe_read_error(ws)
    if status != 0:
        raise RuntimeError(f"device error in the timed region: {status}")
    return {"ms_per_step": ms_per_step, "stage_ms": stage_ms, "touched": touched,
            "weight_set": weight_set, "flush": flush if flush_buf is not None else None,
            "flush_bytes": 2 * l2_bytes if flush_buf is not None else 0,
            "clocks": clk}


def w13_kernel_name(decode: bool, T: int) -> str:
    if not decode:
        return "grouped_gemm_kernel<0> (w13 + activation)"
    if T <= 8:
        return "decode_w13_few_kernel (w13 + act, cp.async rings, mma.sync)"
    if T <= 64:
        return "decode_tc_kernel<N,0> (w13 + act, tcgen05, split over all SMs)"
    return "decode_w13_kernel (w13 + act)"


def roofline_of(args, shp, m, decode, peaks, peak_src, config_name, fp8=False):
    """Roofline of the dominant kernel, the w13 product with the fused
    activation (2/3 of the layer's FLOPs and of its weight bytes), and the
    whole layer's fraction.  FLOPs count real rows only, bytes count each
    touched expert once.  The w13 product does 2 FLOP per weight byte per
    token routed to the expert; below the ridge point (peak FLOP/s / peak
    B/s) it is bound by streaming the touched experts' weights from HBM."""
    touched = m["touched"]
    w13_ms = m["stage_ms"][3]
    rows = shp.T * shp.k + shp.T * shp.n_shared
    # FP8: one byte per weight, and the e4m3 tensor peak at the nominal 2x of
    # the measured bf16 figure
    wbytes = 1 if fp8 else 2
    tpeak = float(peaks["bf16_tflops"]) * (2.0 if fp8 else 1.0)
    ridge = tpeak * 1e12 / (float(peaks["hbm_gbs"]) * 1e9) * (wbytes / 2.0)
    if rows / max(touched, 1) < ridge:
        achieved = touched * (2.0 * shp.I * shp.H * wbytes) / (w13_ms / 1e3) / 1e9
        peak = float(peaks["hbm_gbs"])
        return {"bound": "hbm",
                "kernel": (("decode_tc_kernel<N,0,F8> (e4m3 w13 + act, tcgen05)" if decode
                            else "grouped_gemm_kernel<0, F8> (e4m3 w13 + activation)")
                           if fp8 else w13_kernel_name(decode, shp.T)),
                "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_source": f"{peak_src} hbm_gbs",
                "traffic": None if fp8 else
                traffic_for(("decode.cu" if shp.T <= 8 else "decode_tc.cu")
                            if decode else "gemm_tc.cu", config_name, args.shape),
                "layer_frac": m["weight_set"] / (m["ms_per_step"] / 1e3) / 1e9 / peak,
                "touched_experts": touched}
    w13_flops = 2.0 * shp.T * (shp.k * shp.I + shp.n_shared * shp.I_shared) * shp.H * 2
    achieved = w13_flops / (w13_ms / 1e3) / 1e12
    peak = tpeak
    return {"bound": "tensor",
            "kernel": ("grouped_gemm_kernel<0, F8> (e4m3 w13 + activation)" if fp8
                       else w13_kernel_name(decode, shp.T)),
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak,
            "peak_source": (f"{peak_src} bf16_tflops (burst) x 2, the nominal e4m3:bf16 "
                            "ratio" if fp8 else f"{peak_src} bf16_tflops (burst)"),
            "traffic": None if fp8 else traffic_for("gemm_tc.cu", config_name, args.shape),
            "layer_frac": shp.flops() / (m["ms_per_step"] / 1e3) / 1e12 / peak}


def launches_per_step(decode: bool, router: bool, fp8: bool = False) -> int:
    # prefill: route, layout x4, gather, two GEMMs, rounding; decode: route,
    # w13, w2, row sum; FP8 adds the two row quantisers on either path
    return (4 if decode else 9) + (2 if fp8 else 0) + (1 if router else 0)


def run_e2e(args, api, inp, s, ws, out, stream, barrier, max_over_ranks,
            flush=None, fp8=None):
    """Same metric through the C ABI with every step's token inputs copied
    from pinned host memory and its output copied back, inside the timed
    region.

    Without ``flush`` the steps are pipelined the way a serving loop runs
    them: the input copies on one stream, moe_forward on the compute stream,
    the output copies on a third, over two device buffers per tensor, so
    that step i+1's inputs and step i-1's output cross PCIe while step i
    computes.  Each step still copies its own inputs in and its own output
    out.  With ``flush`` (an L2 flush; small batches, whose copies are a few
    KB) the flush runs before every step, outside that step's events, the
    steps run one after another, and the step time is the mean of the
    per-step event pairs."""
    import torch
    shp = inp.shape
    dev = inp.x.device
    w8 = fp8_weights(api, fp8) if fp8 is not None else None

    def forward(x_d, z_d, o_d, **kw):
        if w8 is not None:
            api.moe_forward_fp8(s, x_d, z_d, w8, inp.scale, o_d, ws, **kw)
        else:
            api.moe_forward(s, x_d, z_d, inp.w13, inp.w2, inp.scale, inp.w13_sh,
                            inp.w2_sh, o_d, ws, **kw)

    x_h = inp.x.cpu().pin_memory()
    z_h = inp.logits.cpu().pin_memory()
    h2d = x_h.numel() * x_h.element_size() + z_h.numel() * z_h.element_size()
    d2h = shp.T * shp.H * 2
    if flush is not None:
        out_h = torch.empty(shp.T, shp.H, dtype=torch.bfloat16).pin_memory()
        x_d = torch.empty_like(inp.x)
        z_d = torch.empty_like(inp.logits)

        def e2e_step():
            x_d.copy_(x_h, non_blocking=True)
            z_d.copy_(z_h, non_blocking=True)
            forward(x_d, z_d, out)
            out_h.copy_(out, non_blocking=True)

        for _ in range(max(args.warmup, 3)):
            e2e_step()
        torch.cuda.synchronize()
        e0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        e1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush(i)
            e0[i].record(stream)
            e2e_step()
            e1[i].record(stream)
        torch.cuda.synchronize()
        barrier()
        total = sum(a.elapsed_time(b) for a, b in zip(e0, e1))
        return max_over_ranks(total) / args.steps, h2d, d2h

    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    x_d = [torch.empty_like(inp.x) for _ in range(2)]
    z_d = [torch.empty_like(inp.logits) for _ in range(2)]
    o_d = [torch.empty_like(out) for _ in range(2)]
    out_h = [torch.empty(shp.T, shp.H, dtype=torch.bfloat16).pin_memory()
             for _ in range(2)]

    def run(n):
        """n pipelined steps; returns (start event, end event)."""
        ev = lambda: torch.cuda.Event()  # noqa: E731
        ev_in = [ev() for _ in range(n)]
        ev_c = [ev() for _ in range(n)]
        ev_out = [ev() for _ in range(n)]
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_c[i - 2])  # step i-2 has read buffer b
                x_d[b].copy_(x_h, non_blocking=True)
                z_d[b].copy_(z_h, non_blocking=True)
                ev_in[i].record(s_in)
            with torch.cuda.stream(stream):
                stream.wait_event(ev_in[i])
                if i >= 2:
                    stream.wait_event(ev_out[i - 2])  # output buffer b copied out
                forward(x_d[b], z_d[b], o_d[b], stream=stream)
                ev_c[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c[i])
                out_h[b].copy_(o_d[b], non_blocking=True)
                ev_out[i].record(s_out)
        t1.record(s_out)  # after the last output copy, hence after every step
        return t0, t1

    run(max(args.warmup, 3))
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t0, t1 = run(args.steps)
    torch.cuda.synchronize()
    barrier()
    return max_over_ranks(t0.elapsed_time(t1)) / args.steps, h2d, d2h


def other_config_entry(args, api, inputs, name, dev, stream, peaks, peak_src):
    """One line of the ``configs`` key: the same device-timed measurement,
    roofline and CPU-baseline leg (with its parity comparison) for another
    workload, one GPU.  A name ending in +fp8 runs that workload with FP8
    experts (moe_forward_fp8)."""
    import torch
    fp8 = name.endswith("+fp8")
    base_name = name[:-4] if fp8 else name
    inp = inputs.make_inputs(base_name, seed=args.seed, device=dev)
    shp = inp.shape
    fpw = inputs.fp8_experts(shp, seed=args.seed + 1, device=dev) if fp8 else None
    if fp8:  # the bf16 weights are not used
        inp.w13 = inp.w2 = inp.w13_sh = inp.w2_sh = None
    s = api.shape_from(shp)
    ws = api.alloc_workspace_fp8(s, dev) if fp8 else api.alloc_workspace(s, dev)
    out = torch.empty(shp.T, shp.H, dtype=torch.bfloat16, device=dev)
    path = api.PATH_AUTO
    decode = shp.T <= api.DECODE_MAX_T
    m = timed_steps(args, api, inp, s, ws, out, stream, path, None, lambda: None,
                    lambda v: v, sample_clocks_gpu=dev.index or 0, fp8=fpw)
    roof = roofline_of(args, shp, m, decode, peaks, peak_src, name, fp8=fp8)
    gpu = gpu_result(api, inp, s, path, args, fp8=fpw)
    base, parity = cpu_baseline_leg(inp, gpu, budget_s=1.5, fp8=fpw)
    entry = {"workload": workload_name(base_name, shp) +
                         (" with FP8 (e4m3) experts, per-row scales" if fp8 else ""),
             "path": "decode" if decode else "prefill",
             "ms_per_step": m["ms_per_step"],
             "value": shp.T / (m["ms_per_step"] / 1e3), "unit": UNIT,
             "roofline": roof, "layer_frac": roof["layer_frac"],
             "stage_ms": dict(zip(api.STAGE_NAMES, m["stage_ms"])),
             "l2": "flushed before every step" if m["flush"] is not None
                   else "weights far larger than L2",
             "parity": parity, "cpu_baseline": base, "clocks": m["clocks"],
             "gpu_launches": launches_per_step(decode, False, fp8) * args.steps}
    del inp, ws, out, fpw
    torch.cuda.empty_cache()
    return entry


OTHER_CONFIGS = ("many_small_prefill", "skewed_shared_prefill", "decode_t1",
                 "decode_t4", "decode_t16", "decode_t64", "decode_t256",
                 "mixtral_prefill+fp8", "many_small_prefill+fp8", "decode_t4+fp8",
                 "decode_t16+fp8", "decode_t64+fp8")


def run_ours(args):
    import torch
    import torch.distributed as dist

    from mixture_experts_ffn_06_b200 import api, inputs

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev,
                                timeout=__import__("datetime").timedelta(seconds=120))

    inp = make_workload(args, dev, args.seed + rank)
    shp = inp.shape
    s = api.shape_from(shp)
    fpw = inputs.fp8_experts(shp, seed=args.seed + 1 + rank, device=dev) \
        if args.fp8 else None
    if fpw is not None:  # the bf16 weights are not used
        inp.w13 = inp.w2 = inp.w13_sh = inp.w2_sh = None
        torch.cuda.empty_cache()
    ws = api.alloc_workspace_fp8(s, dev) if args.fp8 else api.alloc_workspace(s, dev)
    out = torch.empty(shp.T, shp.H, dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    # all work on a side stream (CUDA graphs are captured off the default one)
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)

    path = {"auto": api.PATH_AUTO, "prefill": api.PATH_PREFILL,
            "decode": api.PATH_DECODE}[args.path]
    decode = path == api.PATH_DECODE or (path == api.PATH_AUTO
                                         and shp.T <= api.DECODE_MAX_T)
    if args.fp8 and decode and shp.T > 64:
        raise SystemExit("--fp8: the decode path takes FP8 experts up to 64 tokens")

    router = None
    if args.router:
        rg = torch.Generator(device=dev).manual_seed(args.seed + 1000 + rank)
        router = (*inputs.router_inputs(shp.T, shp.H, shp.E, rg, dev), 1e-6)

    def barrier():
        if world > 1:
            dist.barrier()

    max_over_ranks = max_over_ranks_fn(world, dev)
    m = timed_steps(args, api, inp, s, ws, out, stream, path, router, barrier,
                    max_over_ranks, sample_clocks_gpu=local, fp8=fpw)
    ms_per_step, stage_ms = m["ms_per_step"], m["stage_ms"]
    flush = m["flush"]

    # ---- the router kernel alone (--router): L2 flushed before each launch
    router_stats = None
    if router is not None:
        l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
        rz = torch.empty(shp.T, shp.E, dtype=torch.float32, device=dev)
        fl = torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev)
        for _ in range(3):
            api.moe_router_logits(s, *router, rz, stream=stream)
        rev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for i, (ra, rb) in enumerate(rev):
            with torch.cuda.stream(stream):
                fl.fill_(i & 0xFF)
            ra.record(stream)
            api.moe_router_logits(s, *router, rz, stream=stream)
            rb.record(stream)
        torch.cuda.synchronize()
        r_ms = max_over_ranks(statistics.mean(ra.elapsed_time(rb) for ra, rb in rev))
        # residual rows, GateLinear weight and scale read; logits written
        r_bytes = (shp.T * shp.H + shp.E * shp.H + shp.H) * 2 + shp.T * shp.E * 4
        router_stats = {"kernel": "router_logits_kernel (RMSNorm, scale, GateLinear)",
                        "us": r_ms * 1e3, "bytes": r_bytes,
                        "achieved_gbs": r_bytes / (r_ms / 1e3) / 1e9,
                        "tflops": 2.0 * shp.T * shp.H * shp.E / (r_ms / 1e3) / 1e12,
                        "timing": "L2 flushed before each launch"}
        del fl

    # ---- end to end: pinned host inputs in, host output back, every step
    e2e_ms, h2d, d2h = run_e2e(
        args, api, inp, s, ws, out, stream, barrier, max_over_ranks, flush, fp8=fpw) \
        if not (args.profile or args.router) else (None, 0, 0)

    result = None
    if rank == 0:
        peaks, peak_src = load_peaks()
        value = whole_job_rate(shp.T, world, ms_per_step)
        roof = roofline_of(args, shp, m, decode, peaks, peak_src, args.config,
                           fp8=args.fp8)
        layer_tflops = shp.flops() / (ms_per_step / 1e3) / 1e12
        cpu = parity = None
        if world == 1 and not args.profile:
            gpu = gpu_result(api, inp, s, path, args, fp8=fpw)
            cpu, parity = cpu_baseline_leg(inp, gpu, budget_s=12.0, fp8=fpw)
        weight_set = m["weight_set"]
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3 experts, bf16 activations" if args.fp8 else "bf16",
            "data": "synthetic: seeded N(0,1) tokens, N(0,0.02) bf16 random-init "
                    "expert weights, fp32 router logits with a 1e-3 top-k margin",
            "config": {"workload": workload_name(args.config, shp)
                                   + (" with FP8 (e4m3) experts, per-row scales"
                                      if args.fp8 else ""),
                       "path": "decode" if decode else "prefill",
                       "combine": "fixed-order" if (decode or args.deterministic)
                                  else "fp32 reductions",
                       "timing": ("one CUDA-graph replay of the K steps"
                                  if not args.no_graph else "stream launches")
                                 + ("; step time = mean of per-step event pairs"
                                    if flush is not None else ""),
                       "global_batch": world * shp.T, "seq_len": shp.T,
                       "parallelism": "replicas" if world > 1 else "single",
                       "l2": (f"L2 flushed before every step ({m['flush_bytes'] / 1e6:.0f}"
                              " MB write outside the step's events): the step "
                              f"touches {weight_set / 1e6:.0f} MB of expert weights"
                              if flush is not None else
                              "inputs larger than L2: the step streams the "
                              f"{weight_set / 1e9:.2f} GB of the {m['touched']} "
                              "experts it routes to")},
            "roofline": roof,
            "layer_tflops": layer_tflops,
            "stage_ms": dict(zip(api.STAGE_NAMES, stage_ms)),
            "cpu_baseline": cpu,
            "parity": parity,
            "e2e": None if e2e_ms is None else
                   {"value": world * shp.T / (e2e_ms / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "timing": "steps one after another, L2 flushed before each"
                              if flush is not None else
                              "pipelined: input copies, moe_forward and output "
                              "copies on three streams, two buffers each"},
            "gpu_launches": launches_per_step(decode, router is not None, args.fp8) *
                            args.steps,
            "clocks": m["clocks"],
        }
        if router_stats is not None:
            router_stats["frac_hbm"] = router_stats["achieved_gbs"] / float(peaks["hbm_gbs"])
            result["router"] = router_stats
            result["config"]["workload"] += " + router (from hidden states)"
        if world == 1 and not args.profile and not args.router and not args.shape \
                and args.config == "mixtral_prefill" and not args.headline_only \
                and not args.fp8:
            # the other workloads of the benchmark, one GPU each, after the
            # headline: device time, roofline, parity against the oracle
            del inp, ws, out, fpw
            torch.cuda.empty_cache()
            result["configs"] = {
                name: other_config_entry(args, api, inputs, name, dev, stream, peaks,
                                         peak_src)
                for name in OTHER_CONFIGS}
            result["gpu_launches"] += sum(c["gpu_launches"]
                                          for c in result["configs"].values())
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


# ---------------------------------------------------------- reference arm

def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    import numpy as np
    import torch
    import oracle
    from mixture_experts_ffn_06_b200 import inputs

    inp = make_workload(args, "cpu", args.seed)
    shp = inp.shape
    cores = oracle.num_threads()
    per_step = min(cores, shp.T)
    xu, w13u, w2u = oracle._u16(inp.x), oracle._u16(inp.w13), oracle._u16(inp.w2)
    sh13, sh2 = oracle._u16(inp.w13_sh), oracle._u16(inp.w2_sh)
    rng = np.random.default_rng(1)

    def step():
        tok = rng.choice(shp.T, per_step, replace=False)
        oracle.forward(xu, inp.logits, w13u, w2u, shp.k, shp.act,
                       scale=inp.scale, w13_sh=sh13, w2_sh=sh2, tokens=tok,
                       nthreads=per_step)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    secs = time.perf_counter() - t0
    value = per_step * args.steps / secs
    sample = (f"{per_step} tokens per step drawn from the {shp.T}-token batch, "
              f"full layer per token in fp64")
    result = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same recipe and seed as the CUDA arm)",
        "config": {"workload": workload_name(args.config, shp),
                   "global_batch": shp.T, "seq_len": shp.T,
                   "parallelism": "single"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": per_step,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)
    return result


def run_block(args):
    """The Gemma 4 MoE block (moe_gemma4_block) on the config's MoE shape
    with a dense MLP of intermediate size args.block: K steps in one CUDA
    graph, device-timed, the L2 flushed before every step when the touched
    weights would fit in it.  One GPU; prints one JSON line."""
    import torch

    from mixture_experts_ffn_06_b200 import api, inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = make_workload(args, dev, args.seed)
    shp = inp.shape
    Id = args.block
    blk = inputs.gemma4_block_inputs(shp.T, shp.H, shp.E, Id, seed=args.seed + 7,
                                     device=dev)
    s = api.shape_from(shp)
    ws = api.alloc_gemma4_workspace(s, Id, dev)
    out = torch.empty(shp.T, shp.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)

    def step():
        api.moe_gemma4_block(s, blk.x, blk.norms, 1e-6, blk.mlp_w13, blk.mlp_w2,
                             blk.router_w, blk.router_scale, 1e-6, inp.w13, inp.w2,
                             inp.scale, out, ws, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    weights = 3.0 * shp.H * (shp.I * min(shp.E, shp.T * shp.k) + Id) * 2
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=dev) if weights < 4 * l2 else None
    # external events: captured as event-record nodes that stay timeable
    # after the replay
    ev = [(torch.cuda.Event(enable_timing=True, external=True),
           torch.cuda.Event(enable_timing=True, external=True))
          for _ in range(args.steps)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
    g.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    clocks.begin()
    g.replay()
    torch.cuda.synchronize()
    clocks.end()
    clk = clocks.stop()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    flops = shp.flops() + 6.0 * shp.T * shp.H * Id
    peaks, src = load_peaks()
    print(json.dumps({
        "metric": "Gemma 4 MoE block tokens/s (dense MLP + MoE + norms, 1 B200)",
        "value": shp.T / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_name(args.config, shp) + f" + dense I={Id}",
                   "l2": "flushed before every step" if flush is not None
                   else "weights far larger than L2"},
        "tflops": flops / (ms / 1e3) / 1e12,
        "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / float(peaks["bf16_tflops"]),
        "peak_source": src, "clocks": clk}), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.block:
        run_block(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
