"""Benchmark of the GDR-2 chunkwise forward on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one gdr2_forward call over the 1.3B-layer workload (B=4, H=16,
T=4096, d_k=d_v=128, chunk 64, bf16 q/k/v/b/w, fp32 log-decay and state),
with every input resident in HBM. The step's inputs (541 MB read + written)
are larger than L2 (126 MB), so successive steps cannot reuse cached data.

N > 1 runs one process per GPU (torchrun); every rank processes its own batch
of independent (batch, head) recurrences (weak scaling, no collective on the
data path) and the step time is the maximum over ranks.

The JSON line carries:
  value / ms_per_step  device time of K timed steps (CUDA events on the launch stream)
  e2e                  same metric through the C ABI with pinned HOST buffers:
                       host->device copy of the inputs, the forward, device->host
                       copy of o and S_T, all inside the timed region
  roofline             HBM roofline of the forward call (algorithmic bytes / time); at
                       this size the call is one kernel, the fused chunk-and-scan launch
  tensor               algorithmic FLOP/s against the dense bf16 peak
  components           decode step (256 seq x 16 heads, fp32 state), backward
                       (B=2, T=4096, with and without saved states), the sequence-length
                       sweep (65,536 tokens per call, T = 2048 .. 32768), packed sequences,
                       scalar (KDA) gates, the block's output epilogue and prologue, each
                       with its own figures
  cpu_baseline         the fp64 oracle on the host cores (rank 0, N = 1)
  clocks               SM clocks and throttle reasons sampled during the timed region
`--impl reference` times the oracle itself on the same workload (sampled heads).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_wy_b200 import inputs as I  # noqa: E402

METRIC = "GDR-2 chunk fwd tokens/s at H=16,d=128 (1×B200) and % tensor-core peak"
WORKLOAD = "gdr2_forward B=4 H=16 T=4096 dk=dv=128 C=64 bf16 (1.3B-model layer)"
BYTES_PER_TOKEN_HEAD = 3 * 256 + 512 + 2 * 256 + 256  # q,k,v bf16 + log_alpha fp32 + b,w bf16 + o bf16
FLOP_PER_TOKEN_HEAD = 139_264  # chunk products at C=64, d=128, triangular parts counted once
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
LAUNCHES_PER_STEP = 1  # the fused forward kernel (chunk tasks, then the scans), after a memset of its flags


# ----------------------------------------------------------------------------- distributed plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world > 1 and not dist.is_initialized():
        import datetime

        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def barrier(world: int):
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch of independent recurrences."""
    return base + 7 * rank


def job_throughput(local_total_ms: float, steps: int, units_per_rank: int, world: int, device):
    """Whole-job units/s: every rank's units over the slowest rank's time.

    Returns (units per second, ms per step of the slowest rank)."""
    total_ms = max_over_ranks(local_total_ms, world, device)
    ms_per_step = total_ms / steps
    return units_per_rank * world / (ms_per_step * 1e-3), ms_per_step


# ----------------------------------------------------------------------------- measurement helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_wy_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.startswith("fwd_") or f.endswith(".cuh"):
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def committed_record(kernel: str):
    """The committed ncu record of a kernel (DRAM bytes per launch, device-time shares), if it
    was captured from this source; None otherwise."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f).get(kernel)
    if not d or d.get("source_sha") != kernel_source_sha():
        return None
    return d


class ClockSampler:
    """SM clock and clock-event (throttle) reasons polled through NVML every ~2 ms
    while the timed region runs (reading only; no setting is touched)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = None

    def _handle(self, nv):
        try:
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def __enter__(self):
        import threading

        try:
            import pynvml as nv

            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                    bits = int(get_reasons(h))
                    self.reasons.update(n for b, n in self.REASONS.items() if bits & b)
                except Exception:
                    pass
                self._stop.wait(0.002)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def time_steps(fn, steps: int, stream) -> list:
    """Per-step device times (ms), CUDA events recorded on the launching stream."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for s, e in evs:
        s.record(stream)
        fn()
        e.record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in evs]


def time_steps_queued(fn, steps: int, stream) -> list:
    """time_steps for calls whose host-side work (argument checks, output allocation) can
    outlast their kernels: the stream first spins on the device long enough for every step
    to be enqueued, so the events see the kernels back to back, not the host's pace."""
    torch.cuda._sleep(200_000_000)  # about 0.1 s at the B200's clock
    return time_steps(fn, steps, stream)


# ----------------------------------------------------------------------------- the oracle (CPU baseline)
def oracle_tokens_per_s(x: I.FwdInputs, heads, nthreads):
    """Time the fp64 oracle on the listed (batch, head) recurrences over the full T."""
    import numpy as np

    import oracle

    B, T, H, dk = x.q.shape
    n = x.as_numpy64()
    sel = {f: np.ascontiguousarray(np.stack([n[f][b, :, h] for b, h in heads], axis=1)[None])
           for f in ("q", "k", "v", "log_alpha", "b", "w")}
    t0 = time.perf_counter()
    oracle.forward(sel["q"], sel["k"], sel["v"], sel["log_alpha"], sel["b"], sel["w"], nthreads=nthreads)
    dt = time.perf_counter() - t0
    return len(heads) * T / H / dt, dt


# ----------------------------------------------------------------------------- arms
def run_reference(args, world, rank):
    """The oracle as it stands, on the host cores, with this bench's metric and workload."""
    if rank != 0:
        return
    cfg = I.FWD_1P3B_BF16
    x = I.make_forward_inputs(**cfg)
    B, T, H = cfg["B"], cfg["T"], cfg["H"]
    heads = [(b, h) for b in range(B) for h in range(H)][:16]  # a quarter of the workload per step
    nthr = cores()
    for _ in range(args.warmup):
        oracle_tokens_per_s(x, heads[:2], nthr)
    times = []
    for _ in range(args.steps):
        _, dt = oracle_tokens_per_s(x, heads, nthr)
        times.append(dt)
    tok = len(heads) * T / H
    value = tok * len(times) / sum(times)
    sample = f"{len(heads)} of {B * H} (batch, head) recurrences over the full T={T} per step (fp64, OpenMP)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthr, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def bench_components(dev, stream, peaks):
    """Decode step and backward timings (each with its own roofline); not part of the step."""
    from gated_delta_rule_wy_b200 import gdr2_backward, gdr2_decode_step, gdr2_forward

    out = {}
    cfg = I.DECODE_1P3B
    N, H, dk, dv = cfg["N"], cfg["H"], cfg["dk"], cfg["dv"]
    gen = torch.Generator(device=dev).manual_seed(cfg["seed"])
    S = torch.randn((N, H, dk, dv), device=dev, generator=gen) * cfg["state_std"]
    pool = [I.make_token_inputs((N, H, dk), (N, H, dv), cfg["dtype"], cfg["decay_shift"], gen) for _ in range(8)]
    o = torch.empty((N, H, dv), dtype=cfg["dtype"], device=dev)
    it = [0]

    def dec():
        gdr2_decode_step(*pool[it[0] % 8], S, out=o)
        it[0] += 1

    for _ in range(5):
        dec()
    ms = time_steps_queued(dec, 200, stream)
    us = 1e3 * statistics.median(ms)
    state_bytes = 2 * N * H * dk * dv * 4
    tok_bytes = N * H * (3 * dk * 2 + dk * 4 + 2 * dv * 2 + dv * 2)  # q,k,b bf16 + log_alpha + v,w + o
    gbs = (state_bytes + tok_bytes) / (us * 1e-6) / 1e9
    out["decode"] = {"workload": "256 seq x 16 heads, d=128, fp32 state 256 MiB, one token per call",
                     "us_per_step": us, "tokens_per_s": N / (us * 1e-6), "gbs": gbs,
                     "hbm_frac": gbs / peaks["hbm_gbs"]}
    del S, pool
    cfg = I.BWD_1P3B_BF16
    x = I.make_forward_inputs(**cfg).to(dev)
    dO = I.make_upstream_grad(cfg["B"], cfg["T"], cfg["H"], cfg["dv"], cfg["seed"], dtype=cfg["dtype"]).to(dev)
    _, _, saved = gdr2_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, None, save_states=True)
    from gated_delta_rule_wy_b200 import gdr2_backward_workspace_bytes
    wsb = torch.empty(gdr2_backward_workspace_bytes(cfg["B"], cfg["T"], cfg["H"], cfg["dk"], cfg["dv"], cfg["dtype"]),
                      dtype=torch.uint8, device=dev)
    use = [saved]

    def bwd():
        gdr2_backward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, dO, None, None, use[0], workspace=wsb)

    for _ in range(3):
        bwd()
    t = statistics.median(time_steps_queued(bwd, 10, stream))
    use[0] = None  # the chunk-entry states recomputed inside the call
    for _ in range(2):
        bwd()
    t_re = statistics.median(time_steps_queued(bwd, 10, stream))
    th = cfg["B"] * cfg["T"] * cfg["H"]
    nchunks = cfg["B"] * cfg["H"] * ((cfg["T"] + 63) // 64)
    state = cfg["dk"] * cfg["dv"] * 4
    # per token-head: q, k, v, b, w, dO read and dq, dk, dv, db, dw written in bf16, log alpha read
    # and dlog alpha written in fp32 (3840 B at d = 128); the saved chunk states read; dS0 written
    alg = th * (11 * 128 * 2 + 2 * 128 * 4) + nchunks * state + cfg["B"] * cfg["H"] * state
    out["backward"] = {"workload": "B=2 H=16 T=4096 d=128 bf16, saved chunk states (recompute: without)",
                       "ms_per_call": t, "tokens_per_s": cfg["B"] * cfg["T"] / (t * 1e-3),
                       "algorithmic_bytes": alg, "hbm_frac": alg / (t * 1e-3) / 1e9 / peaks["hbm_gbs"],
                       "ms_per_call_recompute": t_re}
    del x, dO, saved, wsb
    # sequence-length sweep: 65,536 tokens per call at every T (B = 65536 / T), C1 laws
    from gated_delta_rule_wy_b200 import gdr2_forward_workspace_bytes
    sweep = []
    for T in I.SWEEP_T:
        c = I.sweep_config(T)
        xs = I.make_forward_inputs(**c).to(dev)
        o = torch.empty_like(xs.v)
        ws = torch.empty(gdr2_forward_workspace_bytes(c["B"], c["T"], c["H"], c["dk"], c["dv"], c["dtype"]),
                         dtype=torch.uint8, device=dev)

        def fwd():
            gdr2_forward(xs.q, xs.k, xs.v, xs.log_alpha, xs.b, xs.w, None, out=o, workspace=ws)

        for _ in range(3):
            fwd()
        ms = statistics.median(time_steps_queued(fwd, 10, stream))
        tokens = c["B"] * T
        alg = tokens * c["H"] * BYTES_PER_TOKEN_HEAD + c["B"] * c["H"] * c["dk"] * c["dv"] * 4
        sweep.append({"T": T, "B": c["B"], "ms_per_call": ms, "tokens_per_s": tokens / (ms * 1e-3),
                      "hbm_frac": alg / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]})
        del xs, o, ws
    out["sweep"] = {"workload": "65,536 tokens per call, H=16, d=128, bf16, T = 2048 .. 32768", "points": sweep}
    # packed sequences: the same 65,536 tokens cut at 63 distinct random points into 64 sequences
    import numpy as np

    from gated_delta_rule_wy_b200 import gdr2_forward_varlen, gdr2_forward_varlen_workspace_bytes, gdr2_sync_status
    rng = np.random.default_rng(1007)
    cuts = np.sort(rng.choice(np.arange(1, I.SWEEP_TOKENS), size=63, replace=False))
    lens = np.diff(np.concatenate([[0], cuts, [I.SWEEP_TOKENS]]))
    Tt = int(lens.sum())
    xs = I.make_forward_inputs(B=1, H=16, T=Tt, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0,
                               seed=1007).to(dev)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
    o = torch.empty((Tt, 16, 128), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(gdr2_forward_varlen_workspace_bytes(len(lens), Tt, 16, 128, 128), dtype=torch.uint8,
                     device=dev)

    def fwd_packed():
        gdr2_forward_varlen(xs.q, xs.k, xs.v, xs.log_alpha, xs.b, xs.w, cu, None, out=o, workspace=ws)

    for _ in range(3):
        fwd_packed()
    ms = statistics.median(time_steps_queued(fwd_packed, 10, stream))
    gdr2_sync_status()
    out["packed"] = {"workload": f"{Tt} tokens as {len(lens)} packed sequences (random cuts; lengths "
                                 f"{int(lens.min())} .. {int(lens.max())}), H=16, d=128, bf16",
                     "ms_per_call": ms, "tokens_per_s": Tt / (ms * 1e-3)}
    del xs, o, ws
    # the 1.3B-layer forward with KDA / Gated DeltaNet gates: b = w = beta, one value per token-head
    c = I.FWD_1P3B_BF16
    xs = I.make_forward_inputs(**c).to(dev)
    beta = torch.sigmoid(torch.randn((c["B"], c["T"], c["H"]), generator=torch.Generator().manual_seed(1008)))
    beta = beta.to(c["dtype"]).to(dev)
    o = torch.empty_like(xs.v)
    ws = torch.empty(gdr2_forward_workspace_bytes(c["B"], c["T"], c["H"], c["dk"], c["dv"], c["dtype"]),
                     dtype=torch.uint8, device=dev)

    def fwd_kda():
        gdr2_forward(xs.q, xs.k, xs.v, xs.log_alpha, beta, beta, None, out=o, workspace=ws)

    for _ in range(3):
        fwd_kda()
    ms = statistics.median(time_steps_queued(fwd_kda, 20, stream))
    gdr2_sync_status()
    tokens = c["B"] * c["T"]
    alg = tokens * c["H"] * (BYTES_PER_TOKEN_HEAD - 2 * 256 + 2 * 2) + c["B"] * c["H"] * c["dk"] * c["dv"] * 4
    out["kda_gates"] = {"workload": "B=4 H=16 T=4096 d=128 bf16 with b = w = beta scalar per token-head",
                        "ms_per_call": ms, "tokens_per_s": tokens / (ms * 1e-3),
                        "algorithmic_bytes": alg, "hbm_frac": alg / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del xs, o, ws, beta
    # the same forward followed by the block's output epilogue (RMSNorm and SiLU gate) as its own pass
    xs = I.make_forward_inputs(**c).to(dev)
    g, wt = I.make_epilogue_inputs((c["B"], c["T"], c["H"], c["dv"]), c["dv"], seed=1009)
    g, wt = g.to(dev), wt.to(dev)
    o = torch.empty_like(xs.v)
    ws = torch.empty(gdr2_forward_workspace_bytes(c["B"], c["T"], c["H"], c["dk"], c["dv"], c["dtype"]),
                     dtype=torch.uint8, device=dev)

    def fwd_epi():
        gdr2_forward(xs.q, xs.k, xs.v, xs.log_alpha, xs.b, xs.w, None, out=o, workspace=ws, out_gate=g,
                     norm_weight=wt)

    for _ in range(3):
        fwd_epi()
    ms = statistics.median(time_steps_queued(fwd_epi, 20, stream))
    gdr2_sync_status()
    alg = tokens * c["H"] * (BYTES_PER_TOKEN_HEAD + 2 * c["dv"]) + c["B"] * c["H"] * c["dk"] * c["dv"] * 4
    out["epilogue"] = {"workload": "B=4 H=16 T=4096 d=128 bf16, output RMSNorm x weight x SiLU(gate) as "
                                   "a pass after the forward",
                       "ms_per_call": ms, "tokens_per_s": tokens / (ms * 1e-3),
                       "algorithmic_bytes": alg, "hbm_frac": alg / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del xs, o, ws, g, wt
    # the block prologue in front of that forward: short convolutions + SiLU (+ L2) and the
    # decay and gate activations, from the projections' outputs
    from gated_delta_rule_wy_b200 import gdr2_block_prologue
    pin = {k: v.to(dev) for k, v in I.make_prologue_inputs(c["B"], c["T"], c["H"], c["dk"], c["dv"], 4, c["dtype"],
                                                             seed=1010).items()}

    def prologue():
        gdr2_block_prologue(pin["xq"], pin["xk"], pin["xv"], pin["conv_q"], pin["conv_k"], pin["conv_v"], pin["a"],
                            pin["b"], pin["w"])

    for _ in range(3):
        prologue()
    ms = statistics.median(time_steps_queued(prologue, 20, stream))
    gdr2_sync_status()
    th = tokens * c["H"]
    # per token-head: q, k, v read and written in bf16; a read in bf16, log alpha written in fp32;
    # b and w read and written in bf16 (3328 B at d = 128)
    alg = th * (2 * (2 * c["dk"] + c["dv"]) * 2 + c["dk"] * (2 + 4) + 4 * (c["dk"] + c["dv"]))
    out["prologue"] = {"workload": "B=4 H=16 T=4096 d=128 bf16: q, k = L2(SiLU(conv4(x))), v = SiLU(conv4(x)), "
                                   "log alpha = -softplus(a), b, w = sigmoid",
                       "ms_per_call": ms, "tokens_per_s": tokens / (ms * 1e-3), "algorithmic_bytes": alg,
                       "hbm_frac": alg / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del pin
    return out


def run_ours(args, world, rank, local):
    from gated_delta_rule_wy_b200 import build, gdr2_forward, gdr2_forward_workspace_bytes, gdr2_sync_status

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    if rank == 0 or world == 1:
        build.build()
    barrier(world)
    peaks, peak_src = load_peaks()
    cfg = dict(I.FWD_1P3B_BF16)
    cfg["seed"] = shard_seed(cfg["seed"], rank)
    x_cpu = I.make_forward_inputs(**cfg)
    x = x_cpu.to(dev)
    B, T, H, dk, dv = cfg["B"], cfg["T"], cfg["H"], cfg["dk"], cfg["dv"]
    o = torch.empty((B, T, H, dv), dtype=cfg["dtype"], device=dev)
    ws = torch.empty(max(1, gdr2_forward_workspace_bytes(B, T, H, dk, dv, cfg["dtype"])), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()

    def step():
        gdr2_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, None, out=o, workspace=ws)

    for _ in range(args.warmup):
        step()
    gdr2_sync_status()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms = time_steps(step, args.steps, stream)
    barrier(world)
    torch.cuda.synchronize()
    gdr2_sync_status()
    tokens = B * T  # per rank
    value, ms_per_step = job_throughput(sum(ms), args.steps, tokens, world, dev)

    # ---- end to end through the C ABI with host buffers ----
    pinned = [t.pin_memory() for t in (x_cpu.q, x_cpu.k, x_cpu.v, x_cpu.log_alpha, x_cpu.b, x_cpu.w)]
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    sT_host = torch.empty((B, H, dk, dv), dtype=torch.float32).pin_memory()
    dbufs = [torch.empty_like(t, device=dev) for t in pinned]
    h2d = sum(t.numel() * t.element_size() for t in pinned)
    d2h = o_host.numel() * o_host.element_size() + sT_host.numel() * 4

    def e2e_step():
        for d, hsrc in zip(dbufs, pinned):
            d.copy_(hsrc, non_blocking=True)
        oo, sT, _ = gdr2_forward(*dbufs, None, out=o, workspace=ws)
        o_host.copy_(oo, non_blocking=True)
        sT_host.copy_(sT, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 10))
    barrier(world)
    e2e_value, _ = job_throughput(sum(time_steps(e2e_step, e2e_steps, stream)), e2e_steps, tokens, world, dev)

    # ---- roofline of the forward kernel (one launch per step) ----
    alg_bytes = B * T * H * BYTES_PER_TOKEN_HEAD + B * H * dk * dv * 4
    alg_flop = B * T * H * FLOP_PER_TOKEN_HEAD
    t_launch = statistics.mean(ms) * 1e-3
    achieved = alg_bytes / t_launch / 1e9
    rec = committed_record("fwd")
    traffic = float(rec["dram_bytes_per_launch"]) if rec else None
    # the call's kernels and their shares of its device time, from the committed ncu record
    kernel = "one gdr2_forward call"
    if rec and "device_time_share" in rec:
        kernel += ": " + " + ".join(f"{k} ({100 * v:.0f}% of its device time under ncu)"
                                    for k, v in rec["device_time_share"].items())
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peak_src,
                "algorithmic_bytes_per_launch": alg_bytes, "kernel": kernel}
    tflops = alg_flop / t_launch / 1e12
    tensor = {"achieved_tflops": tflops, "peak_tflops": peaks["bf16_tflops"],
              "frac": tflops / peaks["bf16_tflops"], "algorithmic_flop_per_launch": alg_flop,
              "attainable_frac": max(alg_bytes / (peaks["hbm_gbs"] * 1e9), alg_flop / (peaks["bf16_tflops"] * 1e12))
              / t_launch}

    comps = None
    cpu = None
    if world == 1:
        comps = bench_components(dev, stream, peaks)
        heads = [(b, h) for b in range(B) for h in range(H)]
        # the whole workload, repeated until about 10 s of CPU work (at most 30 s)
        total_t, reps = 0.0, 0
        while total_t < 10.0 and reps < 64:
            _, dt = oracle_tokens_per_s(x_cpu, heads, cores())
            total_t += dt
            reps += 1
            if total_t + dt > 30.0:
                break
        val = reps * B * T / total_t
        cpu = {"value": val, "unit": "tokens/s", "cores": cores(), "kind": "oracle",
               "sample": f"the whole workload ({B * H} recurrences of T={T}) {reps} times, fp64, {total_t:.1f} s"}
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)",
                "config": {"workload": WORKLOAD, "B": B, "H": H, "T": T, "dk": dk, "dv": dv, "chunk": 64,
                           "global_batch": B * world, "seq_len": T, "parallelism": f"replicas x{world}",
                           "l2": "inputs larger than L2 (541 MB per step vs 126 MB)"},
                "clocks": clk.summary(),
                "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
                "gpu_launches": LAUNCHES_PER_STEP * args.steps, "roofline": roofline, "tensor": tensor, "components": comps,
                "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    barrier(world)
    if world > 1:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
