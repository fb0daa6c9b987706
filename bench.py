"""Benchmark: MoE-layer tokens/s of the Occult-style layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one pass of the whole layer over one batch: top-k routing, BRIM
build, ORI -> SFD -> EPD dispatch, grouped SwiGLU experts (+ shared experts),
per-rank pre-reduce and combine, dispatched-row counter and co-activation
histogram, replayed from one CUDA graph.  Inputs are synthetic (seeded),
already resident in HBM when the timed region starts; L2 is flushed between
steps (a 256 MiB write outside the per-step events).  Under torchrun every rank runs its own batch (independent
problems, no data-path collective: weak scaling); the time is the max over
ranks.

`e2e` is the same metric through moe_layer_forward_host(): the step's
logits and activations come from pinned host memory and the output goes back
to host memory inside the timed region.

`--impl reference` times the CPU oracle (the plain reference implementation
of the layer) on the host cores on a bounded sample of the same workload.

`--shuffle` measures token shuffling across two layers on the correlated
prefill workload: per step, the home rank each token is predicted to need at
the next layer (from its experts at this layer) and the reorder of its rows by
that rank; the line also reports the share of next-layer assignments served
on the token's rank before and after.

`--train` measures the training step instead: moe_layer_forward_train then
moe_layer_backward (gradients of x, of the logits and of every weight, fp32
weight gradients), with the backward expert GEMMs (moe_expert_ffn_backward)
timed on their own for the roofline.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from expert_warp_top_b200 import inputs  # noqa: E402

METRIC = "MoE-layer tokens/s (route+BRIM dispatch+grouped GEMM+combine)"
SHUFFLE_METRIC = ("token-shuffle tokens/s (predicted home rank from the previous layer's experts "
                  "+ reorder of the token rows by home rank)")
TRAIN_METRIC = ("MoE-layer training tokens/s (forward + backward: route, BRIM dispatch, grouped "
                "GEMMs, combine; input, logit and weight gradients)")

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the two routed-expert
# GEMM launches of one layer step, from one ncu capture of that workload's GEMMs, valid
# only while the GEMM sources hash to `src`; otherwise reported as null.
GEMM_TRAFFIC = {"corr_prefill": {"bytes": (8113.1 + 798.7 + 1942.2 + 1579.3) * 1e6,
                                 "src": "16ac570cf420e614"}}


def gemm_src_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("ffn_gemm.cuh", "ffn_gemm_pair.cuh", "tc_ptx.cuh"):
        with open(os.path.join(ROOT, "expert_warp_top_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def gemm_traffic(cfg):
    rec = GEMM_TRAFFIC.get(cfg.name)
    return rec["bytes"] if rec and rec["src"] == gemm_src_hash() else None
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
L2_NOTE = "flushed between steps (256 MiB write outside the per-step events)"


def config_obj(cfg, args) -> dict:
    """The workload as both arms print it (one object, the same keys and values)."""
    mode = "training step" if args.train else "forward"
    return {"workload": f"{cfg.name}: T={cfg.T} d={cfg.d} f={cfg.f} E={cfg.E} k={cfg.k} "
                        f"R={cfg.R} S={cfg.S} ({mode})",
            "T": cfg.T, "d": cfg.d, "f": cfg.f, "E": cfg.E, "k": cfg.k, "R": cfg.R, "S": cfg.S,
            "fs": cfg.fs, "renorm": cfg.renorm, "activations": cfg.dtype,
            "placement": args.placement, "prune_m": args.prune, "l2": L2_NOTE,
            "parallelism": f"{args.gpus} independent replicas"}


def host_inputs(cfg, seed=None):
    """The workload's seeded inputs in host memory.  They are drawn on the GPU
    when one is present, as the GPU arm draws its own, so that the CPU oracle
    sees the same values; on a host without a GPU they are drawn there."""
    if torch.cuda.is_available():
        dev = torch.device("cuda", torch.cuda.current_device())
        inp = inputs.make_inputs(cfg, device=dev, seed=seed)
        out = {k: v.cpu() for k, v in inp.items()}
        del inp
        torch.cuda.empty_cache()
        return out
    return inputs.make_inputs(cfg, device="cpu", seed=seed)


def max_over_ranks(x: float, device) -> float:
    """The largest value of x over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(cfg, rank: int) -> int:
    """Each rank runs its own independent batch (weak scaling): a distinct seed."""
    return cfg.seed + 7919 * rank


def whole_job_tokens_per_s(tokens_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Tokens all ranks processed divided by the slowest rank's time."""
    return world * tokens_per_rank * steps / (max_ms * 1e-3)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"],
                    bf16_sust=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, source="fallback")


# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self.t = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def n_samples(self) -> int:
        return len(self.lines)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.t is not None:
                self.t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
def algorithmic_work(cfg, c_t: int, e_act: int):
    """FLOPs and HBM bytes the layer must spend (not the dense work it avoids)."""
    e = 2 if cfg.dtype == "bf16" else 4
    T, d, f, k, S, fs = cfg.T, cfg.d, cfg.f, cfg.k, cfg.S, cfg.fs
    flops_ffn = 2.0 * 3 * d * f * T * k + 2.0 * 3 * d * fs * T * S
    bytes_ = e * (T * d + c_t * d + c_t * d + 3.0 * e_act * d * f + 3.0 * S * d * fs
                  + c_t * d + c_t * d + T * d) + 4.0 * (T * cfg.E + 4 * T * k + cfg.R * T
                                                         + cfg.L * c_t)
    return flops_ffn, bytes_


def gemm_launches(m_cap: int, G: int, N: int) -> int:
    """Launches of one grouped GEMM: one (CTA pairs or single CTAs, the
    library's own choice; the hybrid two-launch tiling is opt-in)."""
    return 1


def launches_per_step(cfg) -> int:
    # routing + BRIM masks + counter (one kernel), BRIM column scan + histogram 1,
    # BRIM scatter 1, dispatch 1, experts (2 GEMMs), shared experts (2 GEMMs), combine 1
    tk = cfg.T * cfg.k
    n = 1 + 1 + 1 + 1 + 1
    n += gemm_launches(tk, cfg.E, 2 * cfg.f) + gemm_launches(tk, cfg.E, cfg.d)
    if cfg.S:
        F = cfg.S * cfg.fs
        n += gemm_launches(cfg.T, 1, 2 * F) + gemm_launches(cfg.T, 1, cfg.d)
    return n


def train_launches_per_step(cfg) -> int:
    """forward_train (index 3, dispatch, 2 GEMMs, combine) + backward (dispatch of dY,
    2 input-gradient GEMMs, gate-gradient row sum, 2 weight-gradient GEMMs, combine,
    routing backward), shared experts included."""
    tk, f, d = cfg.T * cfg.k, cfg.f, cfg.d
    g = lambda m, G, N: gemm_launches(m, G, N)  # noqa: E731
    n = 3 + 1 + g(tk, cfg.E, 2 * f) + g(tk, cfg.E, d) + 1
    n += 1 + g(tk, cfg.E, f) + g(tk, cfg.E, d) + 1 + 2 + 1 + 1
    if cfg.S:
        F = cfg.S * cfg.fs
        n += 1 + g(cfg.T, 1, 2 * F) + g(cfg.T, 1, d)        # set_two + shared forward
        n += g(cfg.T, 1, F) + g(cfg.T, 1, d) + 2            # shared backward
    return n


def cpu_baseline(cfg, budget_s: float = 12.0, inp=None, slot_of=None):
    """The oracle as it stands, on a bounded sample of the same workload's tokens:
    routing + BRIM build (under the run's placement) + the dense layer on the
    sampled tokens."""
    import oracle
    if inp is None:
        inp = host_inputs(cfg)

    def bits(t):
        t = t.contiguous()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    logits = inp["logits"].numpy()
    x = bits(inp["x"])
    wg, wu, wd = bits(inp["wg"]), bits(inp["wu"]), bits(inp["wd"])
    shared = (bits(inp["sg"]), bits(inp["su"]), bits(inp["sd"])) if cfg.S else None
    slot_of = (np.arange(cfg.E, dtype=np.int32) if slot_of is None
               else np.ascontiguousarray(np.asarray(slot_of, dtype=np.int32)))
    order = np.random.default_rng(0).permutation(cfg.T).astype(np.int32)
    n, total_t, total_n = 8, 0.0, 0
    while total_t < budget_s and total_n < cfg.T:
        tokens = np.sort(order[total_n:total_n + n])
        t0 = time.perf_counter()
        idx, w = oracle.route(np.ascontiguousarray(logits[tokens]), cfg.k, cfg.renorm)
        oracle.brim(idx, w, slot_of, cfg.E, cfg.R)
        oracle.dense_layer(np.ascontiguousarray(x[tokens]), idx, w, wg, wu, wd, shared=shared)
        dt = time.perf_counter() - t0
        total_t += dt
        total_n += len(tokens)
        n *= 2
    return {"value": total_n / total_t, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{total_n} of {cfg.T} tokens (route + BRIM + dense fp64 layer), "
                      f"{total_t:.1f} s"}


def cpu_baseline_train(cfg, budget_s: float = 12.0, inp=None):
    """The oracle's training step on sub-batches of the workload: routing, BRIM
    build, the dense layer and its backward (input, gate and every weight
    gradient, shared experts included) on the first n tokens as a batch."""
    import oracle
    if inp is None:
        inp = host_inputs(cfg)

    def bits(t):
        t = t.contiguous()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    logits = inp["logits"].numpy()
    x = bits(inp["x"])
    wg, wu, wd = bits(inp["wg"]), bits(inp["wu"]), bits(inp["wd"])
    shared = (bits(inp["sg"]), bits(inp["su"]), bits(inp["sd"])) if cfg.S else None
    slot_of = np.arange(cfg.E, dtype=np.int32)
    rng = np.random.default_rng(0)
    total_n, total_t, n = 0, 0.0, 8
    while total_t < budget_s and n <= cfg.T:
        lg = np.ascontiguousarray(logits[:n])
        xs = np.ascontiguousarray(x[:n])
        dy = rng.standard_normal((n, cfg.d))
        t0 = time.perf_counter()
        idx, w = oracle.route(lg, cfg.k, cfg.renorm)
        oracle.brim(idx, w, slot_of, cfg.E, cfg.R)
        oracle.dense_layer(xs, idx, w, wg, wu, wd, shared=shared)
        g = oracle.dense_layer_backward(xs, idx, w, wg, wu, wd, dy, shared=shared,
                                        experts=np.arange(cfg.E), shared_grads=cfg.S > 0)
        oracle.route_backward(lg, idx, g["dw"], cfg.renorm)
        dt = time.perf_counter() - t0
        total_t += dt
        total_n += n
        n *= 2
    return {"value": total_n / total_t, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"sub-batches of the first 8, 16, ... tokens, {total_n} tokens in all "
                      f"(route + BRIM + dense fp64 layer + its backward with every weight "
                      f"gradient), {total_t:.1f} s"}


def oracle_placement(cfg, how):
    """slot_of of the run's placement, computed by the oracle: contiguous, or the
    greedy correlated placement from the co-activation histogram of the same
    calibration batch the GPU arm uses (T = 32768, seed 1)."""
    import oracle
    if how == "contiguous":
        return np.arange(cfg.E, dtype=np.int32)
    calib = cfg.with_(T=32768, seed=1)
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else "cpu"
    logits = inputs.make_logits(calib, device=dev).cpu().numpy()
    idx, _ = oracle.route(logits, calib.k, 0)
    return oracle.place_greedy(oracle.coact_histogram(idx, cfg.E), cfg.R)


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    per_step = []
    budget = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    inp = host_inputs(cfg)
    slot_of = None if args.train else oracle_placement(cfg, args.placement)
    for i in range(args.warmup + args.steps):
        if args.train:
            res = cpu_baseline_train(cfg, budget_s=budget, inp=inp)
        else:
            res = cpu_baseline(cfg, budget_s=budget, inp=inp, slot_of=slot_of)
        if i >= args.warmup:
            per_step.append(res)
    value = statistics.median([r["value"] for r in per_step])
    line = {
        "impl": "reference", "metric": TRAIN_METRIC if args.train else METRIC, "value": value,
        "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * cfg.T / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_obj(cfg, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": per_step[-1]["sample"]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
def run_ours(args, cfg):
    import torch.distributed as dist
    from expert_warp_top_b200 import _binding as B
    from expert_warp_top_b200.layer import MoELayer

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    # each rank: its own independent batch (seed offset by rank), same weights recipe
    inp = inputs.make_inputs(cfg, device=dev, seed=rank_seed(cfg, rank))
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    # the CPU baseline reads these very inputs, copied to host memory
    host_inp = {k_: v.cpu() for k_, v in inp.items()} if want_cpu else None
    slot_of, placement_info = placement(cfg, args.placement, dev, inp["logits"])
    kw = dict(wg=inp.pop("wg"), wu=inp.pop("wu"), wd=inp.pop("wd"))
    if cfg.S:
        kw.update(sg=inp.pop("sg"), su=inp.pop("su"), sd=inp.pop("sd"))
    layer = MoELayer(T=cfg.T, d=cfg.d, f=cfg.f, E=cfg.E, k=cfg.k, R=cfg.R, renorm=cfg.renorm,
                     dtype=inputs.torch_dtype(cfg), S=cfg.S, fs=cfg.fs, slot_of=slot_of,
                     device=dev, prune_m=args.prune, **kw)
    prune_info = None
    if args.prune > 0:
        # the same layer without pruning, once, for C_T and the output deviation
        layer.prune_m = 0
        y_full = layer.forward(inp["logits"], inp["x"]).clone()
        c_t_full = int(layer.c_t.item())
        layer.prune_m = args.prune
        y_pruned = layer.forward(inp["logits"], inp["x"]).float()
        dev_rows = (y_pruned - y_full.float()).abs().amax(1) / y_full.float().abs().amax(1).clamp_min(1e-30)
        prune_info = {"m": args.prune, "c_t_unpruned": c_t_full, "c_t_pruned": int(layer.c_t.item()),
                      "c_t_reduction": 1 - int(layer.c_t.item()) / max(c_t_full, 1),
                      "output_max_row_rel_dev": float(dev_rows.max()),
                      "output_mean_row_rel_dev": float(dev_rows.mean())}
        torch.cuda.synchronize(dev)
    del kw
    logits, x = inp["logits"], inp["x"]
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    # The step is replayed from one CUDA graph, so host launch overhead does not
    # enter the timing.  External event-record nodes inside the graph time the
    # index path (routing, BRIMs, counter, histogram) and the routed-expert
    # GEMMs on their own within every timed step.
    def part_a():
        layer.route_brim(logits)  # routing, BRIMs, counter, histogram
        layer.dispatch(x)

    def part_b():
        layer.experts()

    def part_c():
        layer.shared_experts(x)
        layer.combine()

    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(args.warmup):
            part_a(); part_b(); part_c()
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    status = B.moe_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")
    i0 = torch.cuda.Event(enable_timing=True, external=True)
    i1 = torch.cuda.Event(enable_timing=True, external=True)
    f0 = torch.cuda.Event(enable_timing=True, external=True)
    f1 = torch.cuda.Event(enable_timing=True, external=True)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        i0.record(side)
        layer.route_brim(logits)
        i1.record(side)
        layer.dispatch(x)
        f0.record(side)
        part_b()
        f1.record(side)
        part_c()
    torch.cuda.synchronize(dev)
    c_t = int(layer.c_t.item())
    e_act = int((layer.epd_off[1:] - layer.epd_off[:-1] > 0).sum().item())

    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    step_ms, ffn_ms, index_ms = [], [], []
    with ClockSampler(local_rank) as clocks:
        # keep the GPU busy until the sampler reports, so its samples see the load
        t_end = time.time() + 5.0
        while clocks.n_samples() < 2 and time.time() < t_end:
            for _ in range(20):
                graph.replay()
            torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)  # evict the previous step's working set from L2
            s0.record(stream)
            graph.replay()
            s1.record(stream)
            s1.synchronize()
            step_ms.append(s0.elapsed_time(s1))
            ffn_ms.append(f0.elapsed_time(f1))
            index_ms.append(i0.elapsed_time(i1))
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        # a few more loaded samples after the timed region
        t_end = time.time() + 2.0
        n0 = clocks.n_samples()
        while clocks.n_samples() < n0 + 2 and time.time() < t_end:
            for _ in range(20):
                graph.replay()
            torch.cuda.synchronize(dev)
    status = B.moe_get_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed steps")
    # The routed-expert GEMMs again, alone in a graph of their own (no event
    # nodes between them and their neighbours), on the same EPD rows: the
    # in-step figure above against this one shows what the step's event nodes
    # and neighbours cost the GEMMs.
    g_ffn = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ffn, stream=side):
        part_b()
    torch.cuda.synchronize(dev)
    ffn_own_ms = []
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        s0.record(stream)
        g_ffn.replay()
        s1.record(stream)
        s1.synchronize()
        ffn_own_ms.append(s0.elapsed_time(s1))
    del g_ffn
    total_ms = max_over_ranks(float(sum(step_ms)), dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_tokens_per_s(cfg.T, args.steps, world, total_ms)

    # end to end through the public API: host buffers in and out, copies timed
    e2e = None
    if not args.no_e2e:
        try:
            e2e = e2e_host(layer, inp, cfg, args, dev, world)
        except Exception as exc:  # noqa: BLE001 -- reported, never hidden
            e2e = {"value": None, "unit": UNIT, "error": str(exc)[:200]}

    pk = peaks()
    flops, bytes_ = algorithmic_work(cfg, c_t, e_act)
    # the dominant kernel: the two routed-expert GEMM launches of a step.  Its
    # roofline is the slower of its FLOPs at the bf16 peak and its bytes (the
    # weights of the experts with rows, the A rows, H written and read back,
    # the O rows) at the HBM copy bandwidth.
    e = 2 if cfg.dtype == "bf16" else 4
    ffn_flops = 2.0 * 3 * cfg.d * cfg.f * cfg.T * cfg.k
    ffn_bytes = e * (3.0 * e_act * cfg.d * cfg.f + cfg.T * cfg.k * (cfg.d + 2 * cfg.f + cfg.d))
    ffn_s = statistics.mean(ffn_ms) * 1e-3
    if ffn_bytes / (pk["hbm"] * 1e9) > ffn_flops / (pk["bf16_sust"] * 1e12):
        roof = {"bound": "hbm", "achieved": ffn_bytes / ffn_s / 1e9, "peak": pk["hbm"],
                "unit": "GB/s", "frac": ffn_bytes / ffn_s / 1e9 / pk["hbm"],
                "peak_source": f"{pk['source']} HBM copy bandwidth"}
    else:
        achieved = ffn_flops / ffn_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_sust"],
                "unit": "TFLOP/s", "frac": achieved / pk["bf16_sust"],
                "peak_source": f"{pk['source']} bf16 sustained"}
    roof.update({"kernel": "routed-expert grouped GEMM (gate/up with SwiGLU epilogue + down "
                           "with gate scaling, 2 launches per step)",
                 "algorithmic_flops": ffn_flops, "algorithmic_bytes": ffn_bytes,
                 "traffic": gemm_traffic(cfg)})
    layer_roof_s = max(flops / (pk["bf16_sust"] * 1e12), bytes_ / (pk["hbm"] * 1e9))
    cpu = None
    if want_cpu:
        cpu = cpu_baseline(cfg, inp=host_inp, slot_of=slot_of.cpu().numpy())
        cpu["inputs"] = "the GPU arm's own inputs, copied to host memory"
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype, "data": "synthetic",
            "config": config_obj(cfg, args),
            "placement": placement_info,
            "roofline": roof,
            "layer_roofline": {"t_roof_ms": layer_roof_s * 1e3, "frac": layer_roof_s * 1e3 /
                               ms_per_step, "flops": flops, "bytes": bytes_},
            "c_t": c_t, "tk_rows": cfg.T * cfg.k, "e2e": e2e, "cpu_baseline": cpu,
            "prune": prune_info,
            "clocks": clocks.summary(),
            "gpu_launches": launches_per_step(cfg) * args.steps,
            "ffn_ms": statistics.mean(ffn_ms),
            "ffn_own_graph_ms": statistics.mean(ffn_own_ms),
            "index_ms": statistics.mean(index_ms),
        }
        # the GEMMs' time in SM clock cycles at the median sampled clock: the
        # figure to compare across runs and with ncu at different clocks
        mhz = line["clocks"].get("sm_mhz")
        line["ffn_mcycles"] = line["ffn_ms"] * mhz * 1e-3 if mhz else None
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_train(args, cfg):
    """The training step: moe_layer_forward_train + moe_layer_backward (through
    MoELayer.forward_train / backward), replayed from one CUDA graph; then the
    backward expert GEMMs (moe_expert_ffn_backward) alone for the roofline."""
    import torch.distributed as dist
    from expert_warp_top_b200 import _binding as B
    from expert_warp_top_b200.layer import MoELayer

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    inp = inputs.make_inputs(cfg, device=dev, seed=rank_seed(cfg, rank))
    host_inp = ({k_: v.cpu() for k_, v in inp.items()}
                if rank == 0 and world == 1 and not args.no_cpu_baseline else None)
    kw = dict(wg=inp.pop("wg"), wu=inp.pop("wu"), wd=inp.pop("wd"))
    if cfg.S:
        kw.update(sg=inp.pop("sg"), su=inp.pop("su"), sd=inp.pop("sd"))
    layer = MoELayer(T=cfg.T, d=cfg.d, f=cfg.f, E=cfg.E, k=cfg.k, R=cfg.R, renorm=cfg.renorm,
                     dtype=inputs.torch_dtype(cfg), S=cfg.S, fs=cfg.fs, device=dev, **kw)
    del kw
    logits, x = inp["logits"], inp["x"]
    g = torch.Generator(device=dev).manual_seed(rank_seed(cfg, rank) + 77)
    dy = torch.randn(cfg.T, cfg.d, generator=g, device=dev).to(layer.dtype)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    grads = None

    def step():
        nonlocal grads
        layer.forward_train(logits, x)
        grads = layer.backward(dy, grads=grads)

    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(args.warmup):
            step()
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    if B.moe_get_device_status() != 0:
        raise RuntimeError("device status after warm-up")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step()
    torch.cuda.synchronize(dev)

    # the backward expert GEMMs alone, on the same EPD rows
    layer.route_brim(logits)
    layer.dispatch(x)
    tk, f, d = cfg.T * cfg.k, cfg.f, cfg.d
    a = layer.x_epd if layer.x_epd is not None else layer.x_sfd
    bf = dict(dtype=torch.bfloat16, device=dev)
    z = torch.empty(tk, 2 * f, **bf)
    h = torch.empty(tk, f, **bf)
    o = torch.empty(tk, d, **bf)
    dy_sfd = torch.empty(layer.cap, d, **bf)
    dy_epd = torch.empty(tk, d, **bf) if layer.x_epd is not None else None
    B.moe_dispatch_gather(dy, cfg.k, cfg.R, cfg.L, layer.brim0, layer.brim1, dy_sfd, dy_epd)
    dout = dy_epd if dy_epd is not None else dy_sfd
    B.moe_expert_ffn_train(a, layer.epd_off, layer.w_gu, layer.w_dn, f, layer.epd_gate, z, h, o,
                           m_cap=tk)
    dxe = torch.empty(tk, d, **bf)
    dgate = torch.empty(tk, dtype=torch.float32, device=dev)
    dwg = torch.empty(cfg.E, 2 * f, d, dtype=torch.float32, device=dev)
    dwd = torch.empty(cfg.E, d, f, dtype=torch.float32, device=dev)
    bws = torch.empty(B.moe_expert_ffn_backward_workspace_size(tk, f), dtype=torch.uint8,
                      device=dev)

    def gemm_bwd():
        B.moe_expert_ffn_backward(dout, a, z, layer.epd_off, layer.w_gu, layer.w_dn, f,
                                  layer.epd_gate, dxe, dgate, dwg, dwd, bws, m_cap=tk)

    with torch.cuda.stream(side):
        for _ in range(3):
            gemm_bwd()
    torch.cuda.synchronize(dev)
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=side):
        gemm_bwd()
    torch.cuda.synchronize(dev)

    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    step_ms, bwd_ms = [], []
    with ClockSampler(local_rank) as clocks:
        t_end = time.time() + 5.0
        while clocks.n_samples() < 2 and time.time() < t_end:
            for _ in range(5):
                graph.replay()
            torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            s0.record(stream)
            graph.replay()
            s1.record(stream)
            s1.synchronize()
            step_ms.append(s0.elapsed_time(s1))
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            s0.record(stream)
            g2.replay()
            s1.record(stream)
            s1.synchronize()
            bwd_ms.append(s0.elapsed_time(s1))
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        t_end = time.time() + 2.0
        n0 = clocks.n_samples()
        while clocks.n_samples() < n0 + 2 and time.time() < t_end:
            for _ in range(5):
                graph.replay()
            torch.cuda.synchronize(dev)
    if B.moe_get_device_status() != 0:
        raise RuntimeError("device status after the timed steps")
    total_ms = max_over_ranks(float(sum(step_ms)), dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_tokens_per_s(cfg.T, args.steps, world, total_ms)

    # end to end: the step's logits, x and dy from pinned host memory, dx and
    # d_logits back to pinned host memory, every step (host wall clock)
    h_logits = logits.cpu().pin_memory()
    h_x = x.cpu().pin_memory()
    h_dy = dy.cpu().pin_memory()
    h_dx = torch.empty(cfg.T, cfg.d, dtype=layer.dtype).pin_memory()
    h_dl = torch.empty(cfg.T, cfg.E, dtype=torch.float32).pin_memory()
    d_logits, d_x, d_dy = torch.empty_like(logits), torch.empty_like(x), torch.empty_like(dy)

    def e2e_step():
        d_logits.copy_(h_logits, non_blocking=True)
        d_x.copy_(h_x, non_blocking=True)
        d_dy.copy_(h_dy, non_blocking=True)
        layer.forward_train(d_logits, d_x)
        gr = layer.backward(d_dy, grads=grads)
        h_dx.copy_(gr["dx"], non_blocking=True)
        h_dl.copy_(gr["d_logits"], non_blocking=True)
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        e2e_step()
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        e2e_step()
    e2e_ms = max_over_ranks((time.perf_counter() - t0) * 1e3, dev)
    e2e = {"value": whole_job_tokens_per_s(cfg.T, args.steps, world, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (h_logits, h_x, h_dy)),
           "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in (h_dx, h_dl)),
           "api": "MoELayer.forward_train + backward (moe_layer_forward_train / "
                  "moe_layer_backward), pinned host copies in the step, wall clock"}

    pk = peaks()
    bwd_flops = 2.0 * 6 * d * f * tk          # 2 input-gradient + 2 weight-gradient GEMMs
    step_flops = 2.0 * 9 * d * f * (tk + cfg.T * cfg.S * cfg.fs / max(f, 1))
    bwd_s = statistics.mean(bwd_ms) * 1e-3
    achieved = bwd_flops / bwd_s / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_sust"], "unit": "TFLOP/s",
            "frac": achieved / pk["bf16_sust"], "peak_source": f"{pk['source']} bf16 sustained",
            "kernel": "backward expert GEMMs (moe_expert_ffn_backward: 2 input-gradient GEMMs, "
                      "the first with the SwiGLU/gate backward fused, 2 weight-gradient GEMMs "
                      "with fp32 output, 1 gate-gradient row sum)",
            "algorithmic_flops": bwd_flops, "traffic": None}
    cpu = None
    if host_inp is not None:
        cpu = cpu_baseline_train(cfg, inp=host_inp)
        cpu["inputs"] = "the GPU arm's own inputs, copied to host memory"
    if rank == 0:
        n_launch = train_launches_per_step(cfg)
        line = {
            "metric": TRAIN_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype, "data": "synthetic",
            "config": config_obj(cfg, args),
            "dw_dtype": "fp32",
            "roofline": roof,
            "step_flops": step_flops,
            "step_tflops": step_flops / (ms_per_step * 1e-3) / 1e12,
            "bwd_gemm_ms": statistics.mean(bwd_ms),
            "e2e": e2e, "cpu_baseline": cpu, "clocks": clocks.summary(),
            "gpu_launches": n_launch * args.steps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def cpu_baseline_shuffle(cfg, table, idx1, x, budget_s: float = 10.0):
    """The oracle's shuffle step on growing token prefixes: predicted homes,
    the home-rank order (BRIM_0 over one "expert" per rank) and the row gather."""
    import oracle
    total_n, total_t, n = 0, 0.0, 256
    while total_t < budget_s and n <= cfg.T:
        t0 = time.perf_counter()
        home = oracle.predict_home(np.ascontiguousarray(idx1[:n]), table)
        b = oracle.brim(home[:, None], np.ones((n, 1)), np.arange(cfg.R, dtype=np.int32), cfg.R,
                        cfg.R)
        oracle.gather_rows(np.ascontiguousarray(x[:n]), b["sfd_token"])
        total_t += time.perf_counter() - t0
        total_n += n
        n *= 2
    return {"value": total_n / total_t, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"token prefixes of 256, 512, ... ({total_n} tokens in all): predicted "
                      f"homes, home-rank order, row gather; {total_t:.1f} s"}


def run_shuffle(args, cfg):
    import torch.distributed as dist
    from expert_warp_top_b200 import _binding as B

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    assert cfg.groups > 0, "token shuffling is measured on a workload with planted groups"
    T, E, k, R = cfg.T, cfg.E, cfg.k, cfg.R
    i32 = dict(dtype=torch.int32, device=dev)

    def route(logits):
        idx = torch.empty(logits.shape[0], k, **i32)
        w = torch.empty(logits.shape[0], k, dtype=torch.float32, device=dev)
        B.moe_route_topk(logits, k, cfg.renorm, idx, w)
        return idx

    # calibration batch: layer-(l+1) placement from its co-activation, and the
    # inter-layer affinity of layer-l experts to layer-(l+1) ranks
    c1, c2 = (route(l) for l in inputs.make_layer_pair_logits(cfg.with_(seed=1), device=dev))
    coact = torch.zeros(E, E, **i32)
    B.moe_coact_histogram(c2, E, coact, 0)
    slot2 = B.moe_place_greedy(coact.cpu(), R).to(dev)
    hist = torch.empty(E, E, **i32)
    B.moe_interlayer_histogram(c1, c2, E, hist, 0)
    table = torch.empty(E, R, **i32)
    B.moe_rank_affinity(hist, slot2, R, table)
    # the evaluation batch (this rank's own)
    l1, l2 = inputs.make_layer_pair_logits(cfg, device=dev, seed=rank_seed(cfg, rank))
    idx1, idx2 = route(l1), route(l2)
    g = torch.Generator(device=dev).manual_seed(rank_seed(cfg, rank) + 5)
    x = torch.randn(T, cfg.d, generator=g, device=dev).to(inputs.torch_dtype(cfg))
    home = torch.empty(T, **i32)
    perm = torch.empty(T, **i32)
    rank_off = torch.empty(R + 1, **i32)
    x_out = torch.empty_like(x)
    ws = torch.empty(B.moe_token_shuffle_workspace_size(T, R), dtype=torch.uint8, device=dev)

    def step():
        B.moe_predict_home(idx1, table, home)
        B.moe_token_shuffle(home, R, perm, rank_off, ws, x=x, x_out=x_out)

    stream = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(args.warmup):
            step()
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    if B.moe_get_device_status() != 0:
        raise RuntimeError("device status after warm-up")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        step()
    torch.cuda.synchronize(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    s0 = torch.cuda.Event(enable_timing=True)
    s1 = torch.cuda.Event(enable_timing=True)
    step_ms = []
    with ClockSampler(local_rank) as clocks:
        t_end = time.time() + 5.0
        while clocks.n_samples() < 2 and time.time() < t_end:
            for _ in range(50):
                graph.replay()
            torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            s0.record(stream)
            graph.replay()
            s1.record(stream)
            s1.synchronize()
            step_ms.append(s0.elapsed_time(s1))
        if world > 1:
            dist.barrier()
        t_end = time.time() + 2.0
        n0 = clocks.n_samples()
        while clocks.n_samples() < n0 + 2 and time.time() < t_end:
            for _ in range(50):
                graph.replay()
            torch.cuda.synchronize(dev)
    if B.moe_get_device_status() != 0:
        raise RuntimeError("device status after the timed steps")
    total_ms = max_over_ranks(float(sum(step_ms)), dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_tokens_per_s(T, args.steps, world, total_ms)

    # served on the token's rank at layer l+1: contiguous home vs predicted home
    cnt = torch.empty(2, dtype=torch.int64, device=dev)
    B.moe_count_local(idx2, slot2, E, R, cnt)
    base = cnt.cpu().tolist()
    B.moe_count_local(idx2, slot2, E, R, cnt, home=home)
    shuf = cnt.cpu().tolist()

    # end to end: layer-l experts and rows from pinned host memory, the
    # reordered rows and the order back to pinned host memory
    h_idx1 = idx1.cpu().pin_memory()
    h_x = x.cpu().pin_memory()
    h_out = torch.empty_like(h_x).pin_memory()
    h_perm = torch.empty(T, dtype=torch.int32).pin_memory()
    d_idx1, d_x = torch.empty_like(idx1), torch.empty_like(x)

    def e2e_step():
        d_idx1.copy_(h_idx1, non_blocking=True)
        d_x.copy_(h_x, non_blocking=True)
        B.moe_predict_home(d_idx1, table, home)
        B.moe_token_shuffle(home, R, perm, rank_off, ws, x=d_x, x_out=x_out)
        h_out.copy_(x_out, non_blocking=True)
        h_perm.copy_(perm, non_blocking=True)
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        e2e_step()
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        e2e_step()
    e2e_ms = max_over_ranks((time.perf_counter() - t0) * 1e3, dev)
    e2e = {"value": whole_job_tokens_per_s(T, args.steps, world, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": h_idx1.numel() * 4 + h_x.numel() * h_x.element_size(),
           "d2h_bytes_per_step": h_out.numel() * h_out.element_size() + T * 4,
           "api": "moe_predict_home + moe_token_shuffle (C ABI), pinned host copies in the "
                  "step, wall clock"}

    pk = peaks()
    e = x.element_size()
    # algorithmic bytes: rows read and written once; top-k ids read twice (prediction
    # and order), homes written and read, the order and the BRIM_0 written
    bytes_ = 2.0 * T * cfg.d * e + 4.0 * (T * k + 3 * T + R * T + T)
    achieved = bytes_ / (ms_per_step * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
            "frac": achieved / pk["hbm"], "peak_source": f"{pk['source']} HBM copy bandwidth",
            "kernel": "the shuffle step: predict_home + BRIM passes (k = 1, E = R) + row gather",
            "algorithmic_bytes": bytes_, "traffic": None}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        calib_tab = oracle.rank_affinity(hist.cpu().numpy().astype(np.uint32),
                                         slot2.cpu().numpy(), R)
        xb = x.cpu().view(torch.int16).numpy().view(np.uint16) if x.dtype == torch.bfloat16 \
            else x.cpu().numpy()
        cpu = cpu_baseline_shuffle(cfg, calib_tab, idx1.cpu().numpy(), xb)
    if rank == 0:
        line = {
            "metric": SHUFFLE_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": cfg.dtype, "data": "synthetic",
            "config": {"workload": f"{cfg.name}: T={T} d={cfg.d} E={E} k={k} R={R}, two layers "
                                   f"with planted inter-layer affinity (follow 0.8)",
                       "calibration": "separate batch (seed 1): layer-(l+1) placement from "
                                      "its co-activation, inter-layer affinity table",
                       "l2": "flushed between steps (256 MiB write outside the per-step events)",
                       "parallelism": f"{world} independent replicas"},
            "roofline": roof,
            "served_on_home_rank": {"contiguous_home": base[0] / base[1],
                                    "predicted_home": shuf[0] / shuf[1],
                                    "assignments": base[1]},
            "e2e": e2e, "cpu_baseline": cpu, "clocks": clocks.summary(),
            "gpu_launches": 5 * args.steps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


EP_METRIC = ("expert-parallel MoE-layer tokens/s (route + BRIM + SFD rows out by all-to-all-v "
             "+ destination BRIM/EPD + grouped GEMMs + pre-reduce + return rows by "
             "all-to-all-v + combine)")


def run_ep(args, cfg):
    """Real expert parallelism (expert_warp_top_b200/ep.py).  Under torchrun each
    of the N ranks is an EP rank (R = N) with T / N of the workload's tokens and
    the experts at its slots, exchanging over NCCL; with one process, the
    workload's R ranks run on the one GPU and exchange through loopback copies
    (every rank's kernels and copies on that GPU, one after another)."""
    import datetime
    import torch.distributed as dist
    from expert_warp_top_b200 import _binding as B
    from expert_warp_top_b200.ep import (DistExchange, EPRank, LoopbackExchange, PeerExchange,
                                         ep_forward)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    R = world if world > 1 else cfg.R
    cfg = cfg.with_(R=R)
    if cfg.E % R or cfg.T % R:
        raise SystemExit(f"--ep needs R = {R} to divide E = {cfg.E} and T = {cfg.T}")
    if world > 1:
        if args.exchange == "peer":
            raise SystemExit("--exchange peer holds all ranks in one process (N = 1)")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        ex = DistExchange()
        mine = [rank]
    else:
        ex = PeerExchange(R) if args.exchange == "peer" else LoopbackExchange(R)
        mine = list(range(R))
    L, Tr = cfg.E // R, cfg.T // R
    inp = inputs.make_inputs(cfg, device=dev)  # the same seeded batch and weights on every rank
    slot_of, placement_info = placement(cfg, args.placement, dev, inp["logits"])
    at = torch.empty(cfg.E, dtype=torch.long)
    at[slot_of.long()] = torch.arange(cfg.E)
    ranks, lgs, xs = [], [], []
    for r in mine:
        e = at[r * L:(r + 1) * L].to(dev)
        kw = {}
        if cfg.S:
            kw = dict(S=cfg.S, fs=cfg.fs, sg=inp["sg"], su=inp["su"], sd=inp["sd"])
        ranks.append(EPRank(rank=r, R=R, T=Tr, d=cfg.d, f=cfg.f, E=cfg.E, k=cfg.k,
                            renorm=cfg.renorm, dtype=inputs.torch_dtype(cfg), slot_of=slot_of,
                            wg=inp["wg"][e], wu=inp["wu"][e], wd=inp["wd"][e], device=dev, **kw))
        lgs.append(inp["logits"][r * Tr:(r + 1) * Tr].contiguous())
        xs.append(inp["x"][r * Tr:(r + 1) * Tr].contiguous())
    for key in ("wg", "wu", "wd"):
        inp.pop(key)
    stream = torch.cuda.current_stream(dev)
    names = ("start", "sent", "exchanged", "computed", "returned", "end")
    ev = {n: torch.cuda.Event(enable_timing=True) for n in names}
    marks = lambda n: ev[n].record(stream)  # noqa: E731
    for _ in range(args.warmup):
        ep_forward(ranks, ex, lgs, xs)
    torch.cuda.synchronize(dev)
    if B.moe_get_device_status() != 0:
        raise RuntimeError("device status after warm-up")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    step_ms, phase_ms = [], {n: [] for n in names[1:]}
    with ClockSampler(local_rank) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            ev["start"].record(stream)
            ep_forward(ranks, ex, lgs, xs, marks=marks)
            ev["end"].record(stream)
            ev["end"].synchronize()
            step_ms.append(ev["start"].elapsed_time(ev["end"]))
            prev = "start"
            for n in names[1:]:
                phase_ms[n].append(ev[prev].elapsed_time(ev[n]))
                prev = n
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    if B.moe_get_device_status() != 0:
        raise RuntimeError("device status after the timed steps")
    total_ms = max_over_ranks(float(sum(step_ms)), dev)
    counts = ep_forward.counts
    c_t = sum(sum(row) for row in counts)
    e = 2 if cfg.dtype == "bf16" else 4
    wire = sum(counts[s][q] for s in range(R) for q in range(R) if s != q)
    if rank == 0:
        line = {
            "metric": EP_METRIC, "value": cfg.T * args.steps / (total_ms * 1e-3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": dict(config_obj(cfg, args), parallelism=(
                f"expert parallel over {world} GPUs (NCCL)" if world > 1 else
                f"{R} expert-parallel ranks on one GPU, " + (
                    "rows written straight into the receiving ranks' buffers (peer movers)"
                    if args.exchange == "peer" else "loopback copies for the all-to-all"))),
            "placement": placement_info,
            "ep": {"ranks": R, "c_t": c_t, "rows_between_ranks": wire,
                   "payload_bytes_each_way": wire * cfg.d * e,
                   "phase_ms": {n: statistics.mean(v) for n, v in phase_ms.items()}},
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    del ranks
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def placement(cfg, how, dev, logits):
    """slot_of for the run ("contiguous", or "histogram": correlated placement
    from the expert co-activation histogram of a separate calibration batch,
    T = 32768, seed 1, routed and counted on the GPU and placed by
    moe_place_greedy), and the C_T of the evaluation batch under both
    placements (the counter kernel), whichever the run uses."""
    from expert_warp_top_b200 import _binding as B
    ident = torch.arange(cfg.E, dtype=torch.int32)
    calib = cfg.with_(T=32768, seed=1)
    c_logits = inputs.make_logits(calib, device=dev)
    idx = torch.empty(calib.T, calib.k, dtype=torch.int32, device=dev)
    w = torch.empty(calib.T, calib.k, dtype=torch.float32, device=dev)
    B.moe_route_topk(c_logits, calib.k, 0, idx, w)
    hist = torch.zeros(cfg.E, cfg.E, dtype=torch.int32, device=dev)
    B.moe_coact_histogram(idx, cfg.E, hist, 0)
    slot_hist = B.moe_place_greedy(hist, cfg.R)
    e_idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    e_w = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev)
    B.moe_route_topk(logits, cfg.k, cfg.renorm, e_idx, e_w)
    per = torch.empty(cfg.R, dtype=torch.int32, device=dev)
    tot = torch.empty(1, dtype=torch.int64, device=dev)
    rem = torch.empty(1, dtype=torch.int64, device=dev)
    out = {}
    for name, s in (("contiguous", ident), ("histogram", slot_hist)):
        B.moe_count_dispatched_rows(e_idx, s.to(dev), cfg.E, cfg.R, per, tot, rem)
        out[name] = int(tot.item())
    tk = cfg.T * cfg.k
    info = {"used": how if how == "contiguous" else
            "histogram (calibration batch T=32768, seed 1)",
            "c_t_contiguous": out["contiguous"], "c_t_histogram": out["histogram"],
            "tk_rows": tk,
            "histogram_row_reduction_vs_per_expert": 1 - out["histogram"] / tk,
            "histogram_row_reduction_vs_contiguous": 1 - out["histogram"] / out["contiguous"]}
    return (ident if how == "contiguous" else slot_hist), info


# Batches in flight in the end-to-end measurement (one stream, workspace and
# host output buffer each).  With three, the copies of two batches overlap a
# third's layer, and the small index and mover kernels of one batch can run
# beside another's GEMM on the SMs it leaves free.
E2E_IN_FLIGHT = 3


def e2e_host(layer, inp, cfg, args, dev, world):
    """End to end through the host-buffer C entry points: every step copies that
    step's logits and activations from pinned host memory, runs the whole layer
    and copies y back to pinned host memory (host wall clock).  E2E_IN_FLIGHT
    batches are in flight (moe_layer_forward_host_async on as many streams,
    each with its own workspace and output buffer), so batches' copies overlap
    other batches' layers; a stream is synchronised before its buffers are
    reused and at the end, so every step's y is in host memory inside the timed
    region.  The fully synchronous moe_layer_forward_host is timed too
    ("sync")."""
    import torch.distributed as dist
    h_logits = inp["logits"].cpu().pin_memory()
    h_x = inp["x"].cpu().pin_memory()
    nf = E2E_IN_FLIGHT
    h_ys = [torch.empty(layer.y.shape, dtype=layer.y.dtype).pin_memory() for _ in range(nf)]
    wss = [layer.host_workspace() for _ in range(nf)]
    streams = [torch.cuda.Stream(dev) for _ in range(nf)]

    def pipelined(n):
        for i in range(n):
            s = streams[i % nf]
            s.synchronize()  # the batch nf steps back: its buffers are free, its y is home
            layer.forward_host(h_logits, h_x, h_ys[i % nf], stream=s, ws=wss[i % nf],
                               asynchronous=True)
        for s in streams:
            s.synchronize()

    pipelined(args.warmup)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    pipelined(args.steps)
    ms = max_over_ranks((time.perf_counter() - t0) * 1e3, dev)

    for _ in range(args.warmup):
        layer.forward_host(h_logits, h_x, h_ys[0])
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        layer.forward_host(h_logits, h_x, h_ys[0])
    ms_sync = max_over_ranks((time.perf_counter() - t0) * 1e3, dev)
    h2d = h_logits.numel() * h_logits.element_size() + h_x.numel() * h_x.element_size()
    d2h = h_ys[0].numel() * h_ys[0].element_size()
    return {"value": whole_job_tokens_per_s(cfg.T, args.steps, world, ms), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "api": f"moe_layer_forward_host_async (C ABI), {nf} batches in flight on {nf} "
                   "streams, pinned host buffers, wall clock",
            "sync": {"value": whole_job_tokens_per_s(cfg.T, args.steps, world, ms_sync),
                     "api": "moe_layer_forward_host (one batch at a time)"}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="corr_prefill", choices=sorted(inputs.CONFIGS),
                    help="workload (default: the correlated-routing prefill layer, T=32768, "
                         "d=4096, f=2048, E=64, k=6, R=8: the largest one-GPU workload)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end (host buffers) measurement, e.g. under a profiler")
    ap.add_argument("--placement", default="contiguous", choices=["contiguous", "histogram"])
    ap.add_argument("--shuffle", action="store_true",
                    help="time token shuffling across two layers (correlated prefill workload)")
    ap.add_argument("--ep", action="store_true",
                    help="time the real expert-parallel layer: R = N ranks over NCCL under "
                         "torchrun, or the workload's R ranks on one GPU (loopback)")
    ap.add_argument("--exchange", choices=["collective", "peer"], default="collective",
                    help="--ep with one process: loopback copies standing for the all-to-all, "
                         "or the peer movers that write into the receiving ranks' buffers")
    ap.add_argument("--train", action="store_true",
                    help="time the training step (forward + backward) instead of the forward")
    ap.add_argument("--prune", type=int, default=0,
                    help="routing-score-based collaboration pruning: keep each token's first "
                         "PRUNE ranks (0 = off)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override the workload's T (for profiling a smaller case of the same "
                         "kernels; the line's config names the override)")
    ap.add_argument("--experts", type=int, default=0,
                    help="override the workload's E (R must divide it)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    cfg = inputs.CONFIGS[args.config]
    if args.tokens or args.experts:
        cfg = cfg.with_(name=f"{cfg.name}[T={args.tokens or cfg.T},E={args.experts or cfg.E}]",
                        T=args.tokens or cfg.T, E=args.experts or cfg.E)
    if args.impl == "reference":
        run_reference(args, cfg)
    elif args.train:
        run_train(args, cfg)
    elif args.shuffle:
        run_shuffle(args, cfg)
    elif args.ep:
        run_ep(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
