"""Benchmark of the causal attention backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c4] [--impl reference]

A step is one whole backward pass (attn_bwd: preprocess, main tile loop, dQ
conversion) over one batch of seeded synthetic inputs already resident in
HBM. The default workload is the largest single-GPU configuration: 1
sequence x 4 heads x 262,144 tokens x 64 channels in bf16 (q, k scaled by
0.5). `--config c4` runs 2 x 16 heads x 16,384 tokens x 128 channels. FLOPs
are counted as 2.5x the causal forward's 4*B*H*N^2*d/2.

Statistic: every step is timed by its own CUDA events on the launching
stream; `value` and `ms_per_step` come from the MEDIAN step, the main kernel's
roofline from the median main-kernel time (the means are reported beside
them). A timed region of a second or more runs under the power cap, so the
roofline's peak is then the measured sustained bf16 figure, with the burst
fraction beside it; a shorter region is rated against the burst figure.

Under torchrun each rank runs the same per-GPU workload on its own inputs
(heads are independent; no collective on the data path): weak scaling, value =
all ranks' FLOPs / max-over-ranks device time.

`--impl reference` times the float64 CPU oracle instead (rank 0 only), on a
bounded sample of the same workload per step.

`--layout bnhd|packed` holds the tensors as [B, N, H, d] arrays (packed: q, k,
v in one [B, N, 3, H, d] array, dq, dk, dv in another) and times one
attn_bwd_strided call per step; the roofline then uses that whole call.

`--layer` times one causal multi-head attention layer instead (the attention
sublayer of the nanoGPT-shaped step of ddx issue #217, x [B, N, C] with
C = H*d, the projections as cuBLAS GEMMs, the attention on the strided
kernels): forward + backward per step, FLOPs = 24*B*N*C^2 for the four
projections (forward and both backward products) + the attention's causal
forward and backward.

`--shard-heads` splits ONE problem's (batch, head) pairs over the ranks
(strong scaling; the long-sequence configuration by default): each rank
runs the backward of its block of heads, value = the whole problem's FLOPs
over the slowest rank's step time. `--gather` adds an NCCL all-gather of
dQ, dK, dV to every rank inside the timed step.

`--bob` times the backward-over-backward (fp32 FFMA kernels; the fp32
256-token configuration by default): FLOPs counted as its 12 matrix products
per kept score pair (24*d per pair, 12*B*H*N^2*d causal), against the
derived FFMA peak.

`--rect NQ` times the N_q != N_k backward (attn_bwd_rect): the last NQ
positions of the configuration's N tokens (query row r at position
N - NQ + r) attending causally to all N keys -- the key-value-cache shape --
FLOPs counted over the kept pairs (10*d per pair).

`--block-mask SPEC` (causal, full, window:W, random:P:SEED over 128 x 128
tiles; bf16) times the block-sparse backward instead: the same three stages
with the masked main kernel, FLOPs counted over the kept tiles (a kind-1 tile
as 128 x 128 score pairs, a kind-2 tile as half), so the causal mask gives
the causal count.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from seeded_inputs import CONFIGS, block_mask, block_mask_pairs, draw  # noqa: E402

METRIC = "causal attention backward TFLOP/s (bf16, 1×B200) and % of dense tensor peak"
BOB_METRIC = "causal attention backward-over-backward TFLOP/s (fp32, 1xB200)"
BOB_METRIC_BF16 = "causal attention backward-over-backward TFLOP/s (bf16, 1xB200)"
LAYER_METRIC = "causal multi-head attention layer step TFLOP/s (bf16, forward + backward)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's dense bf16 figure for one B200 (the 2:4-sparse figure halved), for context only
DATASHEET_DENSE_BF16_TFLOPS = 2250.0
MAIN_KERNEL_SOURCE = os.path.join(ROOT, "causal_softmax_attention_b200", "csrc",
                                  "bwd_bf16_sm100.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "bwd_main_dram_traffic.json")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_source_digest() -> str:
    h = hashlib.sha256()
    for name in ("bwd_bf16_sm100.cu", "sm100.cuh", "common.cuh", "tile_walk.cuh"):
        with open(os.path.join(ROOT, "causal_softmax_attention_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def dram_traffic_per_launch(cfg):
    """DRAM bytes per main-kernel launch from the committed ncu summary, scaled
    to this workload by the causal tile pairs processed; None if the summary
    is missing or was taken on a different kernel source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as fh:
        entries = json.load(fh)["captures"]
    digest = kernel_source_digest()
    for t in entries:
        if t.get("kernel_source_digest") == digest and t.get("d") == cfg.d:
            T = math.ceil(cfg.N / 128)
            pairs = cfg.B * cfg.H * T * (T + 1) / 2
            return t["dram_bytes_per_tile_pair"] * pairs
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def __del__(self):
        if self.file is not None and os.path.exists(self.file.name):
            os.unlink(self.file.name)

    def summary(self, t0=None, t1=None):
        """Median SM clock and active throttle reasons of the samples taken
        between host times t0 and t1 (the timed region), or of all samples.
        A timed region shorter than the sampling interval holds no sample:
        then the samples within 0.3 s of it are used, and the result says so."""
        out = self._summary(t0, t1)
        if out.get("samples") == 0 and t0 is not None:
            out = self._summary(t0 - 0.3, t1 + 0.3)
            out["window"] = "timed region +- 0.3 s (the region is shorter than the sampling interval)"
        return out

    def _rows(self):
        if self.proc is None or self.file is None:
            return None
        self.file.flush()
        with open(self.file.name) as fh:
            return [r.strip().split(", ") for r in fh if r.strip()]

    @staticmethod
    def _stamp(field):
        import datetime
        try:
            return datetime.datetime.strptime(field, "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def per_step(self, t_start, step_ms):
        """The median SM clock sampled while each timed step ran, or None for
        a step no sample fell in. The steps run back to back from host time
        t_start (the device is idle when the timed region is enqueued), so
        step s occupies [t_start + sum(step_ms[:s]), + step_ms[s])."""
        rows = self._rows() or []
        samples = []
        for r in rows:
            if len(r) < 9:
                continue
            ts = self._stamp(r[0])
            try:
                samples.append((ts, float(r[1])))
            except ValueError:
                continue
        out, t = [], t_start
        for ms in step_ms:
            t1 = t + ms * 1e-3
            s = [mhz for ts, mhz in samples if ts is not None and t <= ts < t1]
            out.append(statistics.median(s) if s else None)
            t = t1
        return out

    def _summary(self, t0=None, t1=None):
        rows = self._rows()
        if rows is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            ts = self._stamp(r[0])
            if t0 is not None and ts is not None and not (t0 <= ts <= t1):
                continue
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
                power.append(float(r[3]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Maximum of a per-rank time over all ranks (every rank takes part)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Weak scaling: every rank processes its own copy of the workload, so the
    job's throughput is all ranks' FLOPs over the slowest rank's step time."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def sm_count(device=None) -> int:
    """Streaming multiprocessors of the GPU, read at run time."""
    return int(torch.cuda.get_device_properties(device).multi_processor_count)


def ffma_peak_tflops(peaks, device=None) -> float:
    """Derived FP32 FFMA peak: SMs x 128 lanes x 2 FLOP x the maximum SM clock."""
    return sm_count(device) * 128 * 2 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e12


def tensor_peak(peaks, peak_kind: str, timed_seconds: float):
    """(peak, label) for a tensor-core kernel: the sustained bf16 figure when
    the timed region lasts a second or more (the board then sits at its
    power cap), else the burst figure."""
    if timed_seconds >= 1.0 and "bf16_tflops_sustained" in peaks:
        return float(peaks["bf16_tflops_sustained"]), (
            f"{peak_kind} bf16_tflops_sustained (timed region {timed_seconds:.1f} s, "
            "long enough to run under the power cap)")
    return float(peaks["bf16_tflops"]), (
        f"{peak_kind} bf16_tflops (burst; timed region {timed_seconds:.2f} s)")


def clock_bins(step_ms, step_mhz):
    """Steps grouped by the SM clock sampled while they ran (15 MHz bins):
    per bin the step count and median step time, plus the median of
    time x clock (a clock-normalised step length in ms*MHz)."""
    bins = {}
    for ms, mhz in zip(step_ms, step_mhz):
        if mhz is None:
            continue
        key = int(round(mhz / 15.0) * 15)
        bins.setdefault(key, []).append(ms)
    tagged = [ms * mhz for ms, mhz in zip(step_ms, step_mhz) if mhz is not None]
    return {"bins": [{"sm_mhz": k, "steps": len(v), "median_step_ms": statistics.median(v)}
                     for k, v in sorted(bins.items())],
            "steps_with_a_sample": len(tagged),
            "median_ms_x_mhz": statistics.median(tagged) if tagged else None}


# --------------------------------------------------------------------- oracle arms
def oracle_sample(cfg, budget_s: float, rows_per_block: int = 256):
    """Time the float64 oracle on the last query-row blocks of head (0, 0)
    until `budget_s` seconds of CPU work; returns (TFLOP/s, description)."""
    import oracle
    from seeded_inputs import as_f64
    q, k, v, do = draw(1, 1, cfg.N, cfg.d, cfg.seed, cfg.dtype, cfg.qk_gain)
    qh, kh, vh, doh = (as_f64(t[0, 0]) for t in (q, k, v, do))
    flops, elapsed, rows, r1 = 0.0, 0.0, 0, cfg.N
    while elapsed < budget_s:
        if r1 <= 0:  # whole head done: repeat from the end until the budget is spent
            r1 = cfg.N
        r0 = max(0, r1 - rows_per_block)
        t0 = time.perf_counter()
        oracle.backward_row_block(qh, kh, vh, doh, cfg.scale, r0, r1, causal=True)
        elapsed += time.perf_counter() - t0
        pairs = (r1 * (r1 + 1) - r0 * (r0 + 1)) / 2  # causal pairs of rows r0..r1-1
        flops += 10.0 * cfg.d * pairs
        rows += r1 - r0
        r1 = r0
    desc = (f"oracle backward_row_block (numpy float64) on {rows} query rows (last rows first) of one "
            f"head of {cfg.name} (N={cfg.N}, d={cfg.d}): {flops / 10 / cfg.d:.3e} causal pairs "
            f"in {elapsed:.1f} s")
    return flops / elapsed / 1e12, desc, elapsed


def oracle_sample_masked(cfg, spec: str, budget_s: float, n_sample: int = 2048):
    """Time the float64 oracle's block-masked backward on whole heads of
    n_sample tokens with the same mask recipe until `budget_s` seconds of CPU
    work; FLOPs counted over the kept tiles, as on the GPU."""
    import oracle
    from seeded_inputs import as_f64
    n = min(cfg.N, n_sample)
    bm = block_mask(spec, n)
    keep = oracle.block_mask_keep(bm, n)
    q, k, v, do = draw(1, 1, n, cfg.d, cfg.seed, cfg.dtype, cfg.qk_gain)
    qh, kh, vh, doh = (as_f64(t[0, 0]) for t in (q, k, v, do))
    flops, elapsed, heads = 0.0, 0.0, 0
    while elapsed < budget_s:
        t0 = time.perf_counter()
        oracle.backward_head(qh, kh, vh, doh, cfg.scale, keep=keep)
        elapsed += time.perf_counter() - t0
        flops += 10.0 * cfg.d * block_mask_pairs(bm)
        heads += 1
    desc = (f"oracle backward_head (numpy float64, materialised {n}x{n}) with block mask {spec} "
            f"on {heads} heads of {n} tokens, d={cfg.d}, in {elapsed:.1f} s")
    return flops / elapsed / 1e12, desc, elapsed


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample_repeat(name, fn, flops_per_run, budget_s):
    """Run the oracle call `fn` until `budget_s` seconds of CPU work."""
    runs, elapsed = 0, 0.0
    while elapsed < budget_s:
        t0 = time.perf_counter()
        fn()
        elapsed += time.perf_counter() - t0
        runs += 1
    return flops_per_run * runs / elapsed / 1e12, f"{name}: {runs} runs in {elapsed:.1f} s", elapsed


def oracle_c1_single_thread(repeats: int = 5):
    """The oracle's whole backward of the 256-token, 64-channel head (c1,
    fp32 inputs widened to float64) on ONE host thread: the counterpart of
    ddx's ~190 ms of backward steps at 256 tokens x 64 features (an i7-8700,
    12 threads). Median of `repeats` runs, in ms."""
    import oracle
    from seeded_inputs import as_f64
    from threadpoolctl import threadpool_limits
    c = CONFIGS["c1"]
    q, k, v, do = (as_f64(t) for t in draw(c.B, c.H, c.N, c.d, c.seed, c.dtype))
    times = []
    with threadpool_limits(limits=1):
        for _ in range(repeats):
            t0 = time.perf_counter()
            oracle.backward(q, k, v, do, c.scale, True)
            times.append(time.perf_counter() - t0)
    return {"ms": 1e3 * statistics.median(times), "threads": 1, "runs": repeats,
            "workload": "c1: B=1 H=1 N=256 d=64, forward recomputed inside the oracle's backward",
            "context": "ddx's SQL backward steps at 256 tokens x 64 features: about 190 ms "
                       "(i7-8700, 12 threads)"}


def oracle_sample_bob(cfg, budget_s):
    """The double-backward oracle on the whole workload (as the --bob arm)."""
    import oracle
    from seeded_inputs import as_f64
    a = [as_f64(t) for t in draw(cfg.B, cfg.H, cfg.N, cfg.d, cfg.seed, cfg.dtype, cfg.qk_gain)]
    a += [as_f64(t) for t in draw(cfg.B, cfg.H, cfg.N, cfg.d, cfg.seed + 500, cfg.dtype)[:3]]
    return oracle_sample_repeat(
        f"oracle double_backward (numpy float64) on {cfg.name}",
        lambda: oracle.double_backward(*a, cfg.scale, True), 12.0 * cfg.B * cfg.H * cfg.N ** 2 * cfg.d,
        budget_s)


def oracle_sample_layer(cfg, budget_s, n_sample=256):
    """The layer oracle on one sequence of n_sample tokens with the --layer
    arm's widths (C = H*d); FLOPs counted as that arm counts them."""
    import oracle
    from seeded_inputs import as_f64, draw_layer
    C, n = cfg.H * cfg.d, min(cfg.N, n_sample)
    x, wq, wo, dy = (as_f64(t) for t in draw_layer(1, n, C, cfg.seed))
    flops = 24.0 * n * C * C + 7.0 * cfg.H * n * n * cfg.d
    return oracle_sample_repeat(
        f"oracle mha_layer (numpy float64) on 1 x {n} tokens, C={C}, H={cfg.H}",
        lambda: oracle.mha_layer(x, wq, wo, dy, cfg.H), flops, budget_s)


def bob_config(cfg, n_gpus):
    return dict(config_dict(cfg, n_gpus), workload=f"{cfg.name}: causal attention "
                f"backward-over-backward B={cfg.B} H={cfg.H} N={cfg.N} d={cfg.d} {cfg.dtype}, "
                "q,k,v,dO,U ~ N(0,1)" + (f" (q,k x{cfg.qk_gain})" if cfg.qk_gain != 1.0 else ""))


def oracle_sample_bob_prefix(cfg, budget_s, n_sample=1024):
    """The double-backward oracle (materialised, numpy float64) on the first
    n_sample positions of one head -- a causal prefix is itself a causal
    problem -- until `budget_s` seconds of CPU work; FLOPs 12 * n^2 * d."""
    import oracle
    from seeded_inputs import as_f64
    n = min(cfg.N, n_sample)
    a = [as_f64(t[0, 0, :n]) for t in draw(1, 1, cfg.N, cfg.d, cfg.seed, cfg.dtype, cfg.qk_gain)]
    a += [as_f64(t[0, 0, :n]) for t in draw(1, 1, cfg.N, cfg.d, cfg.seed + 500, cfg.dtype)[:3]]
    v, desc, el = oracle_sample_repeat(
        f"oracle double_backward_head (numpy float64, materialised) on the first {n} positions "
        f"of one head of {cfg.name}", lambda: oracle.double_backward_head(*a, cfg.scale, True),
        12.0 * n * n * cfg.d, budget_s)
    return v, desc, el


def layer_config(cfg):
    C = cfg.H * cfg.d
    return {"workload": f"attention layer B={cfg.B} N={cfg.N} C={C} H={cfg.H} (d={cfg.d}), causal, "
                        "x, dy ~ N(0,1), weights ~ N(0,1/C), no biases",
            "B": cfg.B, "N": cfg.N, "C": C, "H": cfg.H, "d": cfg.d, "parallelism": "single GPU",
            "l2": "inputs larger than L2 (no flush needed)"}


RECT_METRIC = "causal attention backward TFLOP/s, N_q < N_k (bf16, 1xB200)"


def rect_pairs(nq: int, nk: int, off: int) -> int:
    """Score pairs the causal filter keeps when query row r is position off + r."""
    r = np.arange(nq, dtype=np.int64)
    return int(np.minimum(nk, off + r + 1).sum())


def rect_config(cfg, nq):
    off = cfg.N - nq
    return {"workload": f"{cfg.name} keys with the last {nq} positions as queries: causal attention "
                        f"backward B={cfg.B} H={cfg.H} N_q={nq} N_k={cfg.N} q_offset={off} "
                        f"d={cfg.d} {cfg.dtype}, q,k,v,dO ~ N(0,1)",
            "B": cfg.B, "H": cfg.H, "N_q": nq, "N_k": cfg.N, "q_offset": off, "d": cfg.d,
            "causal": True, "parallelism": "single GPU",
            "kept_pairs_per_head": rect_pairs(nq, cfg.N, off)}


def mode_metric_config(args, cfg, n_gpus):
    """The metric and config of the measurement the flags select."""
    if args.rect:
        return RECT_METRIC, rect_config(cfg, args.rect)
    if args.bob:
        return (BOB_METRIC_BF16 if cfg.dtype == "bf16" else BOB_METRIC), bob_config(cfg, n_gpus)
    if args.layer:
        return LAYER_METRIC, layer_config(cfg)
    return METRIC, config_dict(cfg, n_gpus, args.block_mask, args.layout)


def run_reference(args, cfg, world, rank):
    if rank != 0:
        return
    budget = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    def sample(b):
        if args.bob:
            return oracle_sample_bob(cfg, b) if cfg.N <= 4096 else oracle_sample_bob_prefix(cfg, b)
        if args.rect:
            return oracle_sample(cfg, b)  # the last query rows of a head: the rectangular problem
        if args.layer:
            return oracle_sample_layer(cfg, b)
        if args.block_mask:
            return oracle_sample_masked(cfg, args.block_mask, b)
        return oracle_sample(cfg, b)

    for _ in range(args.warmup):
        sample(budget / 4)
    vals, descs, times = [], [], []
    for _ in range(args.steps):
        v, d, t = sample(budget)
        vals.append(v)
        descs.append(d)
        times.append(t)
    value = statistics.median(vals)
    cores = blas_threads()
    metric, config = mode_metric_config(args, cfg, args.gpus)
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": descs[-1]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_dict(cfg, n_gpus, mask_spec=None, layout="bhnd"):
    kind = "causal" if mask_spec is None else f"block-sparse ({mask_spec} over 128x128 tiles)"
    if layout != "bhnd":
        kind += f", {layout} layout"
    out = {"workload": f"{cfg.name}: {kind} attention backward B={cfg.B} H={cfg.H} "
                        f"N={cfg.N} d={cfg.d} {cfg.dtype}, q,k,v,dO ~ N(0,1)"
                        + (f" (q,k x{cfg.qk_gain})" if cfg.qk_gain != 1.0 else "")
                        + f", seed {cfg.seed}, scale 1/sqrt(d)",
            "B": cfg.B, "H": cfg.H, "N": cfg.N, "d": cfg.d, "causal": mask_spec is None,
            "global_batch": cfg.B * n_gpus, "seq_len": cfg.N,
            "parallelism": f"independent replicas x{n_gpus}" if n_gpus > 1 else "single GPU",
            "l2": "inputs larger than L2 (no flush needed)"
            if 5 * cfg.B * cfg.H * cfg.N * cfg.d * 2 > 126e6
            else "L2 flushed (256 MB write) between steps, outside the steps' events"}
    out["layout"] = layout
    if mask_spec is not None:
        bm = block_mask(mask_spec, cfg.N)
        out["block_mask"] = mask_spec
        out["kept_fraction_of_causal"] = block_mask_pairs(bm) / (cfg.N * cfg.N / 2)
    return out


# --------------------------------------------------------------------- head-sharded arm
def run_sharded(args, cfg, world, rank, local):
    import causal_softmax_attention_b200 as csa
    from causal_softmax_attention_b200.shard import (backward_shard, gather_heads, head_block,
                                                     head_range)

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, H, N, d = cfg.B, cfg.H, cfg.N, cfg.d
    start, end = head_range(B * H, world, rank)
    nh = end - start
    # every rank draws the same problem and keeps its own heads on the device
    full = draw(B, H, N, d, cfg.seed, cfg.dtype, cfg.qk_gain)
    q, k, v, do = (torch.zeros(B, H, N, d, dtype=t.dtype, device=dev) for t in full)
    for dst, src in zip((q, k, v, do), full):
        if nh:
            head_block(dst, start, end).copy_(head_block(src, start, end))
    del full
    o = torch.zeros_like(q)
    lse = torch.zeros(B, H, N, dtype=torch.float32, device=dev)
    dq, dk, dv = torch.zeros_like(q), torch.zeros_like(k), torch.zeros_like(v)
    stream = torch.cuda.current_stream(dev)
    if nh:
        blk = [head_block(t, start, end) for t in (q, k, v, o, lse)]
        csa.attn_fwd(*blk, True, cfg.scale, stream)
    ws = torch.empty(max(1, csa.attn_bwd_workspace_bytes(1, max(nh, 1), N, d, q.dtype)),
                     dtype=torch.uint8, device=dev)

    def step():
        backward_shard(q, k, v, o, do, lse, dq, dk, dv, ws, world, rank, True, cfg.scale,
                       stream)
        if args.gather and world > 1:
            for t in (dq, dk, dv):
                t.copy_(gather_heads(t, world, rank))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    with ClockSampler(local) as clocks:
        time.sleep(1.0)
        host_t0 = time.time()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        host_t1 = time.time()
        time.sleep(0.25)
    barrier(world)
    ms_per_step = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    flops = cfg.bwd_flops  # the whole problem, shared out
    value = flops / (ms_per_step * 1e-3) / 1e12
    if nh and csa.attn_last_status(ws) != 0:
        raise RuntimeError("device status after the sharded steps")
    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic",
        "config": dict(config_dict(cfg, world), parallelism=f"heads sharded over {world} ranks"
                       + (", dQ/dK/dV all-gathered (NCCL) in the step" if args.gather else "")),
        "roofline": {"bound": "tensor", "achieved": value / world, "peak": peak,
                     "unit": "TFLOP/s", "frac": value / world / peak, "traffic": None,
                     "kernel": "attn_bwd per rank (preprocess, main, dQ convert)"
                               + (" + all-gather" if args.gather else ""),
                     "peak_source": f"{peak_kind} bf16_tflops (burst), per GPU",
                     "algorithmic_flops_per_launch": flops / world, "avg_launch_ms": ms_per_step},
        "e2e": None,
        "gpu_launches": 3 * args.steps,
        "clocks": clocks.summary(host_t0, host_t1),
        "heads_per_rank": -(-(B * H) // world),
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- backward-over-backward arm
def run_bob(args, cfg, world, rank, local):
    import causal_softmax_attention_b200 as csa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, H, N, d = cfg.B, cfg.H, cfg.N, cfg.d
    bf16 = cfg.dtype == "bf16"
    ins = draw(B, H, N, d, cfg.seed + 1000 * rank, cfg.dtype, cfg.qk_gain)
    cots = draw(B, H, N, d, cfg.seed + 1000 * rank + 500, cfg.dtype)[:3]
    host = [t.pin_memory() for t in ins + cots]
    q, k, v, do, uq, uk, uv = (t.to(dev) for t in host)
    o, lse = csa.forward(q, k, v, True, cfg.scale)
    outs = [torch.empty_like(q) for _ in range(4)]
    ws = torch.empty(csa.library().attn_bwd_bwd_workspace_bytes(
        B, H, N, d, csa.ATTN_BF16 if bf16 else csa.ATTN_F32), dtype=torch.uint8, device=dev)
    torch.cuda.reset_peak_memory_stats(dev)
    stream = torch.cuda.current_stream(dev)
    flops = 12.0 * B * H * N * N * d
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def step():
        csa.attn_bwd_bwd(q, k, v, o, do, lse, uq, uk, uv, *outs, ws, True, cfg.scale, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        time.sleep(1.0)
        host_t0 = time.time()
        for i in range(args.steps):
            flush.zero_()  # between steps, outside the step's events
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
        host_t1 = time.time()
        time.sleep(0.25)
    ms_per_step = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / args.steps,
                                 world)
    value = whole_job_tflops(flops, world, ms_per_step)
    # e2e: the seven inputs and O, LSE from pinned host memory, the four
    # gradients back, serialised with the call
    h_o, h_lse = o.cpu().pin_memory(), lse.cpu().pin_memory()
    dev_in, host_in = [q, k, v, do, uq, uk, uv, o, lse], host + [h_o, h_lse]
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]

    def e2e_step():
        for dst, src in zip(dev_in, host_in):
            dst.copy_(src, non_blocking=True)
        step()
        for dst, src in zip(host_out, outs):
            dst.copy_(src, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / args.steps, world)
    if rank != 0:
        return
    if csa.attn_last_status(ws) != 0:
        raise RuntimeError("device status after the double-backward steps")
    peaks, peak_kind = load_peaks()
    if bf16:
        peak, peak_source = tensor_peak(peaks, peak_kind, ms_per_step * args.steps * 1e-3)
        roofline = {"bound": "tensor", "achieved": value / world, "peak": peak, "unit": "TFLOP/s",
                    "frac": value / world / peak, "traffic": None,
                    "kernel": "bob_rows_bf16_kernel + bob_cols_bf16_kernel (+ preprocess)",
                    "peak_source": peak_source,
                    "frac_of_burst": value / world / float(peaks["bf16_tflops"])}
    else:
        ffma = ffma_peak_tflops(peaks, dev)
        roofline = {"bound": "alu", "achieved": value / world, "peak": ffma, "unit": "TFLOP/s",
                    "frac": value / world / ffma, "traffic": None,
                    "kernel": "bob_rows_f32_kernel + bob_cols_f32_kernel (+ preprocess)",
                    "peak_source": f"derived: {sm_count(dev)} SMs x 128 FP32 lanes x 2 FLOP x sm_max_mhz"}
    roofline.update({"algorithmic_flops_per_launch": flops, "avg_launch_ms": ms_per_step,
                     "flops_convention": "12 matrix products per kept pair (24*d), causal N^2/2"})
    line = {
        "metric": BOB_METRIC_BF16 if bf16 else BOB_METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
        "config": bob_config(cfg, world),
        "roofline": roofline,
        "peak_memory_bytes": torch.cuda.max_memory_allocated(dev),
        "memory_per_token_bytes": torch.cuda.max_memory_allocated(dev) / (B * H * N),
        "e2e": {"value": whole_job_tflops(flops, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host_in),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in host_out),
                "ms_per_step": e2e_ms},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks.summary(host_t0, host_t1),
    }
    if world == 1 and not args.no_cpu_baseline:
        if N <= 4096:
            v_cpu, desc, _ = oracle_sample_bob(cfg, args.cpu_seconds)
        else:
            v_cpu, desc, _ = oracle_sample_bob_prefix(cfg, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v_cpu, "unit": "TFLOP/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": desc}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- layer arm
def run_layer(args, cfg, world, rank, local):
    import causal_softmax_attention_b200 as csa
    from causal_softmax_attention_b200 import layer
    from seeded_inputs import draw_layer

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, H, N, d = cfg.B, cfg.H, cfg.N, cfg.d
    C = H * d
    hx, hwq, hwo, hdy = (t.pin_memory() for t in draw_layer(B, N, C, cfg.seed + 1000 * rank))
    x, wq, wo, dy = (t.to(dev) for t in (hx, hwq, hwo, hdy))
    ws = torch.empty(csa.attn_bwd_workspace_bytes(B, H, N, d, x.dtype), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)
    proj = 24.0 * B * N * C * C
    flops = proj + cfg.fwd_flops + cfg.bwd_flops

    def step():
        y, saved = layer.layer_forward(x, wq, wo, H, stream)
        return layer.layer_backward(dy, saved, wq, wo, H, ws, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    with ClockSampler(local) as clocks:
        time.sleep(1.0)
        host_t0 = time.time()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        host_t1 = time.time()
        time.sleep(0.25)
    ms_per_step = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    value = whole_job_tflops(flops, world, ms_per_step)

    # e2e: x, dy and the weights from pinned host memory, dx and the weight
    # gradients back to pinned host memory, serialised with the step
    outs = step()
    host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
    h2d = sum(t.numel() * t.element_size() for t in (hx, hwq, hwo, hdy))
    d2h = sum(t.numel() * t.element_size() for t in host_out)

    def e2e_step():
        for dst, src in zip((x, wq, wo, dy), (hx, hwq, hwo, hdy)):
            dst.copy_(src, non_blocking=True)
        for dst, src in zip(host_out, step()):
            dst.copy_(src, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(1, min(args.steps, 5))
    f0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1) / n_e2e, world)
    if rank != 0:
        return
    if csa.attn_fwd_last_status() != 0:
        raise RuntimeError("forward status after the layer steps")
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    achieved = flops / (ms_per_step * 1e-3) / 1e12
    line = {
        "metric": LAYER_METRIC,
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": layer_config(cfg),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "whole layer step (4 cuBLAS GEMMs x 3 + attention fwd + bwd)",
                     "peak_source": f"{peak_kind} bf16_tflops (burst)",
                     "algorithmic_flops_per_launch": flops, "avg_launch_ms": ms_per_step,
                     "projection_flops": proj},
        "e2e": {"value": whole_job_tflops(flops, world, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": 4 * args.steps,  # attn_fwd, preprocess, main, dQ convert (GEMMs are cuBLAS)
        "clocks": clocks.summary(host_t0, host_t1),
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- rectangular arm
def run_rect(args, cfg, world, rank, local):
    import causal_softmax_attention_b200 as csa
    from seeded_inputs import draw_rect

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, H, nk, d, nq = cfg.B, cfg.H, cfg.N, cfg.d, args.rect
    off = nk - nq
    q, k, v, do = (t.to(dev) for t in draw_rect(B, H, nq, nk, d, cfg.seed + 1000 * rank,
                                                 cfg.dtype))
    o, lse = csa.forward_rect(q, k, v, off, True, cfg.scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = csa.new_workspace(q)
    stream = torch.cuda.current_stream(dev)
    flops = 10.0 * d * B * H * rect_pairs(nq, nk, off)

    def step():
        csa.attn_bwd_rect(q, k, v, o, do, lse, dq, dk, dv, ws, off, True, cfg.scale, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        time.sleep(1.0)
        host_t0 = time.time()
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
        host_t1 = time.time()
        time.sleep(0.25)
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    ms_per_step = max_over_ranks(statistics.median(step_ms), world)
    value = whole_job_tflops(flops, world, ms_per_step)
    if rank != 0:
        return
    if csa.attn_last_status(ws) != 0:
        raise RuntimeError("device status after the rectangular steps")
    peaks, peak_kind = load_peaks()
    peak, peak_source = tensor_peak(peaks, peak_kind, sum(step_ms) * 1e-3)
    line = {
        "metric": RECT_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic", "config": rect_config(cfg, nq),
        "statistic": "median of the timed steps' CUDA-event times (max over ranks)",
        "roofline": {"bound": "tensor", "achieved": value / world, "peak": peak, "unit": "TFLOP/s",
                     "frac": value / world / peak, "traffic": None,
                     "kernel": "attn_bwd_rect (whole call: preprocess, main kernel, dQ convert)",
                     "peak_source": peak_source,
                     "frac_of_burst": value / world / float(peaks["bf16_tflops"]),
                     "algorithmic_flops_per_launch": flops, "avg_launch_ms": ms_per_step,
                     "flops_convention": "10*d per kept pair (5 MMAs)"},
        "e2e": None,
        "gpu_launches": 3 * args.steps,
        "clocks": clocks.summary(host_t0, host_t1),
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- GPU arm
def run_gpu(args, cfg, world, rank, local):
    import causal_softmax_attention_b200 as csa

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    B, H, N, d = cfg.B, cfg.H, cfg.N, cfg.d
    q, k, v, do = draw(B, H, N, d, cfg.seed + 1000 * rank, cfg.dtype, cfg.qk_gain)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    mask = None
    if args.block_mask:
        bm = block_mask(args.block_mask, N)
        mask = torch.from_numpy(bm).to(dev)
        flops = 10.0 * d * block_mask_pairs(bm) * B * H
        fwd_flops = 0.4 * flops
        o = torch.empty_like(qd)
        lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
        csa.attn_fwd_masked(qd, kd, vd, o, lse, mask, cfg.scale)
    else:
        flops, fwd_flops = cfg.bwd_flops, cfg.fwd_flops
        o, lse = csa.forward(qd, kd, vd, True, cfg.scale)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ws = csa.new_workspace(qd)
    stream = torch.cuda.current_stream(dev)
    if args.layout != "bhnd":
        # the same values held in [B, N, H, d] arrays (packed: q, k, v in one
        # [B, N, 3, H, d] array), as [B, H, N, d] views
        def bnhd(x):
            return x.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
        if args.layout == "packed":
            qkv = torch.stack([x.permute(0, 2, 1, 3) for x in (qd, kd, vd)], dim=2).contiguous()
            dqkv = torch.empty_like(qkv)
            sq, sk, sv = (qkv[:, :, c].permute(0, 2, 1, 3) for c in range(3))
            gq, gk, gv = (dqkv[:, :, c].permute(0, 2, 1, 3) for c in range(3))
        else:
            sq, sk, sv = bnhd(qd), bnhd(kd), bnhd(vd)
            gq, gk, gv = bnhd(dq), bnhd(dk), bnhd(dv)
        so, sdo = bnhd(o), bnhd(dod)
    small = 5 * B * H * N * d * 2 <= 126e6
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if small else None

    def step(ev_main=None):
        if args.layout != "bhnd":
            if ev_main is not None:
                ev_main[0].record(stream)
            csa.attn_bwd_strided(sq, sk, sv, so, sdo, lse, gq, gk, gv, ws, True, cfg.scale, stream)
            if ev_main is not None:
                ev_main[1].record(stream)
            return
        csa.attn_bwd_preprocess(o, dod, lse, ws, stream)
        if ev_main is not None:
            ev_main[0].record(stream)
        if mask is None:
            csa.attn_bwd_main(qd, kd, vd, dod, dq, dk, dv, ws, True, cfg.scale, stream)
        else:
            csa.attn_bwd_main_masked(qd, kd, vd, dod, dq, dk, dv, mask, ws, cfg.scale, stream)
        if ev_main is not None:
            ev_main[1].record(stream)
        csa.attn_bwd_dq_convert(dq, ws, cfg.scale, stream)

    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    if csa.attn_last_status(ws) != 0:
        raise RuntimeError("device status after warm-up: " + csa.status_string(csa.attn_last_status(ws)))

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    mains = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        time.sleep(1.0)  # let nvidia-smi start sampling before the timed region
        host_t0 = time.time()
        t_begin = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_begin.record(stream)
        for s in range(args.steps):
            if flush is not None:  # between steps, outside the step's own events
                flush.zero_()
            starts[s].record(stream)
            step(mains[s])
            ends[s].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
        host_t1 = time.time()
        time.sleep(0.25)
    barrier(world)
    total_ms = t_begin.elapsed_time(t_end)
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    main_ms = [a.elapsed_time(b) for a, b in mains]
    step_mhz = clocks.per_step(host_t0, step_ms)
    if flush is not None:
        # the L2 flushes ran between the steps: count the steps' own events
        total_ms = sum(step_ms)
    status = csa.attn_last_status(ws)
    # the median step (each step timed by its own events), max over ranks
    ms_per_step = max_over_ranks(statistics.median(step_ms), world)
    ms_per_step_mean = max_over_ranks(total_ms / args.steps, world)
    value = whole_job_tflops(flops, world, ms_per_step)

    # ---- e2e through the public API with pinned host buffers
    hq, hk, hv, hdo = (t.cpu().pin_memory() for t in (qd, kd, vd, dod))
    hdq, hdk, hdv = (torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (dq, dk, dv))
    d2h = sum(t.numel() * t.element_size() for t in (hdq, hdk, hdv))

    # Host buffers in, host gradients out, through the package's pipelined
    # host path: groups of heads are copied in, differentiated and copied out
    # on three streams, each backward an attn_bwd call of the C ABI.
    e2e_chunks = max(1, min(args.e2e_chunks, B * H))
    ws_chunk = torch.empty(csa.chunk_workspace_bytes(B, H, N, d, qd.dtype, e2e_chunks),
                           dtype=torch.uint8, device=dev)
    dev_bufs = {"q": qd, "k": kd, "v": vd, "o": o, "dout": dod, "lse": lse, "dq": dq, "dk": dk,
                "dv": dv, "workspace": ws_chunk}

    # Two ways through the same public call, both measured: (a) q, k, v, dO
    # cross from the host and O, LSE are recomputed on the device by each
    # head group's forward (FLOPs still counted for the backward only) --
    # the cheaper way when the copies dominate; (b) O and LSE cross too and
    # nothing is recomputed -- the cheaper way when the compute dominates.
    # The faster one is the line's e2e, the other is reported beside it.
    ho, hlse = o.cpu().pin_memory(), lse.cpu().pin_memory()
    h2d_qkvdo = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdo))
    e2e_modes = [
        (lambda: csa.backward_host(hq, hk, hv, None, hdo, None, hdq, hdk, hdv, dev_bufs, True,
                                   cfg.scale, e2e_chunks, stream, block_mask=mask,
                                   recompute_forward=True),
         h2d_qkvdo,
         f"backward_host: pinned host q, k, v, dO in, dQ, dK, dV out, {e2e_chunks} head groups, "
         "H2D / forward + backward / D2H overlapped on three streams (O and LSE recomputed on the "
         "device; the forward's FLOPs are not counted)"),
        (lambda: csa.backward_host(hq, hk, hv, ho, hdo, hlse, hdq, hdk, hdv, dev_bufs, True,
                                   cfg.scale, e2e_chunks, stream, block_mask=mask),
         h2d_qkvdo + ho.numel() * ho.element_size() + hlse.numel() * hlse.element_size(),
         f"backward_host: pinned host q, k, v, O, dO, LSE in, dQ, dK, dV out, {e2e_chunks} head "
         "groups, H2D / backward / D2H overlapped on three streams"),
    ]
    if args.layout != "bhnd":
        # the strided arrays themselves go host -> device -> host around one
        # attn_bwd_strided call (copies serialised with the call)
        dev_in = [x for x in ((qkv,) if args.layout == "packed" else (sq, sk, sv))]
        dev_in = [x if x.is_contiguous() else x.permute(0, 2, 1, 3) for x in dev_in]
        dev_in += [so.permute(0, 2, 1, 3), sdo.permute(0, 2, 1, 3), lse]
        dev_out = [dqkv] if args.layout == "packed" else [x.permute(0, 2, 1, 3) for x in (gq, gk, gv)]
        host_in = [x.cpu().pin_memory() for x in dev_in]
        host_out = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in dev_out]
        d2h = sum(t.numel() * t.element_size() for t in host_out)

        def e2e_step():
            with torch.cuda.stream(stream):
                for dsti, srci in zip(dev_in, host_in):
                    dsti.copy_(srci, non_blocking=True)
                csa.attn_bwd_strided(sq, sk, sv, so, sdo, lse, gq, gk, gv, ws, True, cfg.scale,
                                     stream)
                for dsto, srco in zip(host_out, dev_out):
                    dsto.copy_(srco, non_blocking=True)

        e2e_modes = [(e2e_step, sum(t.numel() * t.element_size() for t in host_in),
                      f"{args.layout} arrays from pinned host memory, one attn_bwd_strided, "
                      "back to host")]

    e2e_steps = max(1, min(args.steps, 5))
    e2e_results = []
    for step_fn, h2d_bytes, path in e2e_modes:
        for _ in range(2):
            step_fn()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            step_fn()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms_m = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
        e2e_results.append({"value": whole_job_tflops(flops, world, e2e_ms_m), "unit": "TFLOP/s",
                            "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h,
                            "ms_per_step": e2e_ms_m, "path": path})
    e2e_results.sort(key=lambda r: -r["value"])

    # ---- the forward that produces O and LSE (not part of the timed step):
    # its own CUDA-event time on the same stream, same inputs, outputs reused.
    fwd_iters = 5

    def fwd():
        if args.layout != "bhnd":
            csa.attn_fwd_strided(sq, sk, sv, so, lse, True, cfg.scale, stream)
        elif mask is None:
            csa.attn_fwd(qd, kd, vd, o, lse, True, cfg.scale, stream)
        else:
            csa.attn_fwd_masked(qd, kd, vd, o, lse, mask, cfg.scale, stream)

    for _ in range(2):
        fwd()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(fwd_iters):
        fwd()
    f1.record(stream)
    torch.cuda.synchronize()
    fwd_ms = max_over_ranks(f0.elapsed_time(f1) / fwd_iters, world)

    if rank != 0:
        return
    peaks, peak_kind = load_peaks()
    main_med = statistics.median(main_ms)
    main_avg = statistics.mean(main_ms)
    achieved = flops / (main_med * 1e-3) / 1e12
    burst = float(peaks["bf16_tflops"])
    peak, peak_source = tensor_peak(peaks, peak_kind, sum(step_ms) * 1e-3)
    traffic = dram_traffic_per_launch(cfg) if mask is None and args.layout == "bhnd" else None
    clk = clocks.summary(host_t0, host_t1)
    clk["per_step"] = clock_bins(step_ms, step_mhz)
    if cfg.dtype == "bf16":
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": traffic,
                    "kernel": "attn_bwd_bf16_sm100_kernel" if args.layout == "bhnd"
                    else "attn_bwd_strided (whole call: preprocess, main kernel, dQ convert)",
                    "peak_source": peak_source,
                    "frac_of_burst": achieved / burst,
                    "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                    "frac_of_datasheet": achieved / DATASHEET_DENSE_BF16_TFLOPS,
                    "datasheet_peak": "NVIDIA dense bf16, 2,250 TFLOP/s (context, not measured)",
                    "statistic": "median main-kernel launch time over the timed steps",
                    "algorithmic_flops_per_launch": flops, "avg_launch_ms": main_med,
                    "mean_launch_ms": main_avg}
    else:
        # the fp32 path runs on the CUDA cores: plain FFMA arithmetic
        ffma = ffma_peak_tflops(peaks, dev)
        roofline = {"bound": "alu", "achieved": achieved, "peak": ffma, "unit": "TFLOP/s",
                    "frac": achieved / ffma, "traffic": None,
                    "kernel": "bwd_dkdv_f32_kernel + bwd_dq_f32_kernel",
                    "peak_source": f"derived: {sm_count(dev)} SMs x 128 FP32 lanes x 2 FLOP x sm_max_mhz",
                    "statistic": "median main-kernel launch time over the timed steps",
                    "algorithmic_flops_per_launch": flops, "avg_launch_ms": main_med,
                    "mean_launch_ms": main_avg}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic", "config": config_dict(cfg, world, args.block_mask, args.layout),
        "statistic": "median of the timed steps' CUDA-event times (max over ranks)",
        "value_mean": whole_job_tflops(flops, world, ms_per_step_mean),
        "ms_per_step_mean": ms_per_step_mean,
        "pct_of_dense_bf16_peak": 100.0 * value / world / burst,
        "roofline": roofline,
        "stage_ms": {"step_median": statistics.median(step_ms), "main_median": main_med,
                     "pre_and_convert_median": statistics.median(step_ms) - main_med},
        "e2e": dict(e2e_results[0], **({"other_path": e2e_results[1]} if len(e2e_results) > 1
                                        else {})),
        "forward": {"kernel": "attn_fwd_bf16_sm100_kernel" if cfg.dtype == "bf16"
                    else "fwd_f32_kernel", "ms": fwd_ms,
                    "tflops": fwd_flops / (fwd_ms * 1e-3) / 1e12,
                    "frac": fwd_flops / (fwd_ms * 1e-3) / 1e12 / roofline["peak"],
                    "flops_convention": "causal forward 4*B*H*N^2*d/2" if mask is None
                    else "4*d per kept score pair (kind-2 tiles count half)",
                    "note": "measured outside the timed backward step"},
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
        "device_status": csa.status_string(status),
        "peak_memory_bytes": torch.cuda.max_memory_allocated(dev),
    }
    if world == 1 and not args.no_cpu_baseline:
        if mask is None:
            v_cpu, desc, _ = oracle_sample(cfg, args.cpu_seconds)
        else:
            v_cpu, desc, _ = oracle_sample_masked(cfg, args.block_mask, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v_cpu, "unit": "TFLOP/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": desc,
                                "c1_single_thread": oracle_c1_single_thread()}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="c5", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=16,
                    help="head groups of the end-to-end (host-buffer) measurement")
    ap.add_argument("--shard-heads", action="store_true",
                    help="split one problem's heads over the ranks (strong scaling)")
    ap.add_argument("--gather", action="store_true",
                    help="with --shard-heads: all-gather dQ, dK, dV inside the step")
    ap.add_argument("--bob", action="store_true",
                    help="time the backward-over-backward (fp32)")
    ap.add_argument("--layer", action="store_true",
                    help="time one attention layer step (projections + attention, fwd + bwd)")
    ap.add_argument("--layout", default="bhnd", choices=["bhnd", "bnhd", "packed"],
                    help="memory layout of q, k, v, o, dO and the gradients")
    ap.add_argument("--rect", type=int, default=0, metavar="NQ",
                    help="time attn_bwd_rect: the last NQ positions as queries over all N keys")
    ap.add_argument("--block-mask", default=None, metavar="SPEC",
                    help="time the block-sparse backward: causal, full, window:W or "
                         "random:P:SEED over 128x128 tiles (bf16 configs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.shard_heads and "--config" not in sys.argv:
        args.config = "c5"  # the long-sequence problem is the one worth sharding
    if args.bob and "--config" not in sys.argv:
        args.config = "c1"  # the fp32 kernels' configuration
    if args.layer and "--config" not in sys.argv:
        args.config = "c4"  # a layer of 16 heads x 128 channels (C = 2048)
    cfg = CONFIGS[args.config]
    if args.rect and (args.rect < 1 or args.rect > cfg.N or args.block_mask or args.bob
                      or args.layer or args.shard_heads or args.layout != "bhnd"):
        ap.error("--rect NQ needs 1 <= NQ <= N and is a measurement of its own")
    if args.layout != "bhnd" and args.block_mask:
        ap.error("--layout and --block-mask are separate measurements")
    if args.block_mask:
        if cfg.dtype != "bf16":
            ap.error("--block-mask needs a bf16 config")
        try:
            block_mask(args.block_mask, 128)  # a malformed spec fails before any GPU work
        except (ValueError, IndexError) as e:
            ap.error(f"--block-mask: {e}")
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, cfg, world, rank)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        if args.layer:
            run_layer(args, cfg, world, rank, local)
        elif args.rect:
            run_rect(args, cfg, world, rank, local)
        elif args.shard_heads:
            run_sharded(args, cfg, world, rank, local)
        elif args.bob:
            run_bob(args, cfg, world, rank, local)
        else:
            run_gpu(args, cfg, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
