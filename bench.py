"""Benchmark: RMA-layer decode tokens/s at batch 512 x 8 layers, and the HBM roofline fraction.

Workload (default): 512 independent sequences, 8 RMA layers, 4 KV groups x 4
query heads, head_dim 256, BF16 K/V; every ring full (1,023 positions) and
every bank full (1,024 records); pending buffers staggered at fill b mod 256
so two sequences per layer admit on every step.  One step = rma_decode_step
for each of the 8 layers (a step that fills a pending buffer runs that
group's admit in the same launch).  Per-step inputs (Q, current K/V,
candidate K/V/score) come from a pool of 16 pre-generated step sets, cycled,
so input generation is outside the timed region.  The 36 GB state is far
larger than L2, so no flush is needed between steps.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
  torchrun --nproc-per-node N bench.py --gpus N ...     (one replica per GPU)
  python bench.py --workload long|ragged|prefill|admit   (other workloads)

Other workloads: "long" = 1 sequence at pos 131,072 (full ring and bank), its
8-layer steps replayed from CUDA graphs, reported with per-step latency median
and p99; "ragged" = random ring/bank/pending fills with 16-level scores
(--batch 32..512); "prefill" = 8 sequences x 8 layers, blocks of 256 from an
empty state, in TFLOP/s; "admit" = the standalone admit of a batch whose
sequences are in phase (every bank and every pending buffer full), in GB/s.
Roofline bytes always come from the exact fills of every timed launch.

Multi-GPU: sequences are independent, so each rank runs its own 512-sequence
replica with no data-path collective ("weak" scaling); the only collectives
are the harness's barrier and the max-over-ranks of the timed duration.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "RMA-layer decode tokens/s at batch 512 x 8 layers; % of B200 HBM roofline"
UNIT = "tokens/s"
# algorithmic bytes per (sequence, layer, decode step) with ring and bank full:
# ring K+V 4*1023*1024, bank K+V 4*1024*1024, q 8192, out 8192, k_cur+v_cur 4096, ring write 4096
BYTES_FULL = 4 * 1023 * 1024 + 4 * 1024 * 1024 + 8192 + 8192 + 4096 + 4096
FALLBACK_HBM_GBS = 6650.0
TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")   # DRAM bytes per launch from ncu captures
# algorithmic bytes of one group's admit: the 1,024 + 256 scores read once, then for every
# admitted candidate its K and V rows (1 KiB together) read from pending and written to the
# bank, and its score written (the two counters written are left out)
ADMIT_SCORE_BYTES = (1024 + 256) * 4
ADMIT_ROW_BYTES = 2 * 1024 + 4


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(name) -> str:
    """First 16 hex digits of the SHA-256 of a kernel's source file (or, for a tuple of names,
    of the files' contents concatenated in that order)."""
    h = hashlib.sha256()
    for n in ((name,) if isinstance(name, str) else name):
        with open(os.path.join(ROOT, "bounded_memory_attention_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """(DRAM bytes per launch, workload it was captured on) for `kernel` ("rma_decode",
    "rma_prefill" or "rma_admit") from profiles/traffic.json, or (None, reason) when there is no
    capture or the kernel's sources changed since it was taken (their hash differs)."""
    if not os.path.exists(TRAFFIC_JSON):
        return None, "no ncu capture"
    with open(TRAFFIC_JSON) as f:
        entry = json.load(f).get(kernel)
    if not entry:
        return None, "no ncu capture"
    if entry.get("kernel_source_sha256_16") != kernel_source_hash(tuple(entry["sources"])):
        return None, "kernel changed since the last ncu capture"
    return int(entry["traffic_bytes_per_launch"]), entry["workload"]


class FillTracker:
    """Algorithmic bytes of every decode launch, from the state's counters tracked on the host
    with the method's counter rules: the step reads min(pos, R) ring rows and bank_fill bank rows
    of every group (1 KiB each, K and V), then pos += 1, pend_fill += 1, and a group whose
    pending buffer fills is admitted (bank_fill = min(A, bank_fill + P), pend_fill = 0).
    Fixed bytes per sequence: q 8,192 + out 8,192 + current K/V 4,096 + ring write 4,096.
    FP8 storage (fp8=True): a K+V row pair is 2 x 256 code bytes + 2 exponent bytes = 514 bytes,
    and the ring write stores 4 groups x 514 bytes."""

    FIXED = 8192 + 8192 + 4096 + 4096
    FIXED_FP8 = 8192 + 8192 + 4096 + 4 * 514

    def __init__(self, counters, R: int = 1023, A: int = 1024, P: int = 256, fp8: bool = False):
        c = counters.astype("int64")
        self.pos, self.bank, self.pend = c[..., 0].copy(), c[..., 1].copy(), c[..., 2].copy()
        self.R, self.A, self.P = R, A, P
        self.row_pair = 514 if fp8 else 1024
        self.fixed = self.FIXED_FP8 if fp8 else self.FIXED

    def launch_bytes(self, layer: int) -> int:
        rows = self.pos[layer].clip(max=self.R) + self.bank[layer]
        return int(rows.sum() * self.row_pair + self.pos.shape[1] * self.fixed)

    def advance(self, layer: int) -> None:
        self.pos[layer] += 1
        self.pend[layer] += 1
        full = self.pend[layer] == self.P
        self.bank[layer] = (self.bank[layer] + self.P * full).clip(max=self.A)
        self.pend[layer][full] = 0

    def step_bytes(self) -> int:
        """Bytes of one step over every layer, then the counters advance."""
        tot = 0
        for layer in range(self.pos.shape[0]):
            tot += self.launch_bytes(layer)
            self.advance(layer)
        return tot


def max_over_ranks(ms: float, world: int, device=None) -> float:
    """The slowest rank's time: every rank calls it with its own device-timed duration
    (the identity for one process)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank: float, ms: float) -> float:
    """Units per second of the whole job: every rank's units over the slowest rank's time."""
    return world * units_per_rank / (ms / 1e3)


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.proc = None
        self.uuid = uuid

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
                pw.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "power_w_max": max(pw),
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# workload set-up (device side)
# ---------------------------------------------------------------------------

def make_decode_workload(rma, torch, si, B: int, L: int, kind: str, seed: int, device, fp8: bool = False):
    """The decode workload's state (BF16; with fp8, the library's quantisation of it into an FP8
    state, the BF16 one then freed), gate parameters and a pool of 16 step inputs."""
    cfg = rma.Config(batch=B, n_layers=L)
    st = rma.State(cfg, device=device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    for name in ("ring_k", "ring_v", "bank_k", "bank_v", "pend_k", "pend_v"):
        getattr(st, name).normal_(generator=g)
    if kind == "ragged":
        for name in ("bank_score", "pend_score"):
            z = torch.randn(getattr(st, name).shape, generator=g, device=device)
            getattr(st, name).copy_((torch.clamp(torch.floor(4 * z) + 8, 0, 15) - 8) / 4)
    else:
        st.bank_score.normal_(generator=g)
        st.pend_score.normal_(generator=g)
    c = si.workload_counters(kind, L, B, cfg.n_groups, seed=seed)
    cnt = torch.zeros(L, B, cfg.n_groups, 4, dtype=torch.int32)
    cnt[..., 0] = torch.from_numpy(c["pos"])
    cnt[..., 1] = torch.from_numpy(c["bank_fill"])
    cnt[..., 2] = torch.from_numpy(c["pend_fill"])
    st.counters.copy_(cnt)
    if fp8:
        cfg8 = rma.Config(batch=B, n_layers=L, kv_format=rma.KV_FP8_E4M3)
        st8 = rma.State(cfg8, device=device)
        rma.state_quantize(st8, st)
        torch.cuda.synchronize(device)
        del st
        torch.cuda.empty_cache()
        cfg, st = cfg8, st8
    w, b = si.gate_params(L, cfg.n_q_heads, cfg.head_dim, seed, device=device)
    pool = [[si.decode_inputs(B, cfg.n_groups, cfg.q_per_group, cfg.head_dim, seed=1000 * s + l, device=device,
                              quantized_scores=(kind == "ragged"))
             for l in range(L)] for s in range(16)]
    torch.cuda.synchronize(device)
    return cfg, st, w, b, pool


def step_input_bytes(B: int, L: int) -> tuple:
    h2d = L * (B * 16 * 256 * 2 + 4 * B * 4 * 256 * 2 + B * 4 * 4)
    d2h = L * B * 16 * 256 * 2
    return h2d, d2h


# ---------------------------------------------------------------------------
# the CPU oracle baseline
# ---------------------------------------------------------------------------

def _np(t):
    """Torch tensor -> numpy in storage form (bf16 as uint16 bits)."""
    import numpy as np
    import torch
    return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()


def cpu_oracle_decode(n_seq: int, n_layers: int, n_steps: int, seed: int = 0) -> dict:
    """Time the oracle on the batch-512 workload restricted to n_seq sequences (one host thread)."""
    import oracle
    import synth_inputs as si
    from threadpoolctl import threadpool_limits
    cfg = oracle.Config(batch=n_seq, n_layers=n_layers)
    cont = si.state_contents(n_layers, n_seq, 4, 256, 1023, 1024, 256, seed=seed)
    c = si.workload_counters("batch", n_layers, n_seq, 4)
    st = oracle.state_from_arrays(cfg, {k: _np(v) for k, v in cont.items()}, **c)
    w, b = si.gate_params(n_layers, 16, 256, seed)
    w, b = w.numpy(), b.numpy()
    ins = [[{k: _np(v) for k, v in si.decode_inputs(n_seq, 4, 4, 256, seed=1000 * s + l).items()}
            for l in range(n_layers)] for s in range(n_steps)]
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        for s in range(n_steps):
            for l in range(n_layers):
                x = ins[s][l]
                oracle.decode_step(st, l, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                   x["cand_score"], w[l], b[l])
                oracle.admit(st, l)
        dt = time.perf_counter() - t0
    return {"value": n_seq * n_steps / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n_seq} of the 512 sequences x {n_layers} layers x {n_steps} steps "
                      f"(decode + admit), FP64 numpy oracle, 1 thread; {dt:.1f} s", "cpu": host_cpu()}


def _usable_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_decode_worker(seq: int, n_layers: int, n_steps: int, start, results) -> None:
    """One process of the all-core baseline: one sequence of the batch-512 workload through
    n_steps decode steps of n_layers layers (decode + admit), one thread; reports its seconds."""
    import oracle
    import synth_inputs as si
    from threadpoolctl import threadpool_limits
    cfg = oracle.Config(batch=1, n_layers=n_layers)
    cont = si.state_contents(n_layers, 1, 4, 256, 1023, 1024, 256, seed=seq)
    c = si.workload_counters("batch", n_layers, 1, 4)
    c["pos"] += seq % 256
    c["pend_fill"] += seq % 256
    st = oracle.state_from_arrays(cfg, {k: _np(v) for k, v in cont.items()}, **c)
    w, b = si.gate_params(n_layers, 16, 256, seq)
    w, b = w.numpy(), b.numpy()
    ins = [[{k: _np(v) for k, v in si.decode_inputs(1, 4, 4, 256, seed=1000 * s + l + 7 * seq).items()}
            for l in range(n_layers)] for s in range(n_steps)]
    start.wait()
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        for s in range(n_steps):
            for l in range(n_layers):
                x = ins[s][l]
                oracle.decode_step(st, l, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                   x["cand_score"], w[l], b[l])
                oracle.admit(st, l)
        results.put(time.perf_counter() - t0)


def _oracle_prefill_worker(seq: int, n_blocks: int, start, results) -> None:
    """One process of the all-core prefill baseline: steady-state blocks of one sequence and layer."""
    import oracle
    import synth_inputs as si
    from threadpoolctl import threadpool_limits
    cfg = oracle.Config(batch=1, n_layers=1)
    cont = si.state_contents(1, 1, 4, 256, 1023, 1024, 256, seed=seq)
    st = oracle.state_from_arrays(cfg, {k: _np(v) for k, v in cont.items()}, pos=4096, bank_fill=1024, pend_fill=0)
    w, b = si.gate_params(1, 16, 256, seq)
    xs = [{k: _np(v) for k, v in si.prefill_inputs(1, 256, 4, 4, 256, seed=100 * seq + j).items()}
          for j in range(n_blocks)]
    start.wait()
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        for x in xs:
            oracle.prefill_block(st, 0, x["q"], x["k"], x["v"], x["cand_k"], x["cand_v"], x["cand_score"],
                                 w[0].numpy(), b[0].numpy())
        results.put(time.perf_counter() - t0)


def _all_cores(target, args_of, n_proc: int) -> float:
    """Run target(*args_of(i), start, results) in n_proc spawned processes (spawn: the parent may
    hold a CUDA context), release them together once all are set up, and return the seconds
    from the release until the last one finishes its timed work."""
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    start, results = ctx.Event(), ctx.Queue()
    procs = [ctx.Process(target=target, args=(*args_of(i), start, results)) for i in range(n_proc)]
    for p in procs:
        p.start()
    time.sleep(0.5)
    # wait until every worker has built its inputs (they block on `start` with little CPU use)
    deadline = time.time() + 300
    while time.time() < deadline and any(p.is_alive() for p in procs):
        import psutil
        busy = sum(psutil.Process(p.pid).cpu_percent(interval=0.2) > 20 for p in procs if p.is_alive())
        if busy == 0:
            break
    t0 = time.perf_counter()
    start.set()
    for _ in procs:
        results.get(timeout=600)
    dt = time.perf_counter() - t0
    for p in procs:
        p.join(timeout=60)
    return dt


def cpu_oracle_decode_allcores(n_steps: int = 2, n_layers: int = 8) -> dict:
    """The oracle on every usable host core: one process per core, each one sequence of the
    batch-512 workload through n_steps steps of n_layers layers; tokens/s over all of them."""
    n = _usable_cores()
    dt = _all_cores(_oracle_decode_worker, lambda i: (i, n_layers, n_steps), n)
    return {"value": n * n_steps / dt, "unit": UNIT, "cores": n, "kind": "oracle",
            "sample": f"{n} of the 512 sequences (one process per core) x {n_layers} layers x {n_steps} steps "
                      f"(decode + admit), FP64 numpy oracle; {dt:.1f} s", "cpu": host_cpu()}


def cpu_oracle_prefill_allcores(n_blocks: int = 2) -> dict:
    """The oracle on every usable host core: one process per core, each steady-state blocks of
    its own sequence at one layer; algorithmic GFLOP/s over all of them."""
    n = _usable_cores()
    dt = _all_cores(_oracle_prefill_worker, lambda i: (i, n_blocks), n)
    flops = prefill_flops(1, 1, 256, 20)[-1] * n_blocks * n
    return {"value": flops / dt / 1e9, "unit": "GFLOP/s", "cores": n, "kind": "oracle",
            "sample": f"{n} sequences (one process per core) x {n_blocks} blocks of 256 tokens at one layer (ring and "
                      f"bank full, forced admits), FP64 numpy oracle; {dt:.1f} s", "cpu": host_cpu()}


def all_and_one_core(all_cores, one_core, unit: str) -> dict:
    """The cpu_baseline object: the oracle on every usable host core (its value and core count),
    with the one-thread figure beside it.  A failure is reported, never a reason to lose the line."""
    out = {"value": None, "unit": unit, "cores": _usable_cores(), "kind": "oracle", "sample": "", "cpu": host_cpu()}
    try:
        out.update(all_cores())
    except Exception as ex:
        out["sample"] = f"all-core run failed: {ex}"
    try:
        out["one_core"] = one_core()
    except Exception as ex:
        out["one_core"] = {"value": None, "unit": unit, "cores": 1, "sample": f"failed: {ex}"}
    return out


def host_cpu() -> str:
    """The host CPU's model name and logical core count."""
    model = "unknown CPU"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return f"{model}, {os.cpu_count()} logical cores"


def cpu_oracle_prefill(seed: int = 0) -> dict:
    """Time the oracle on steady-state prefill blocks (ring and bank full) of one sequence at one
    layer, in algorithmic GFLOP/s (one host thread)."""
    import oracle
    import synth_inputs as si
    from threadpoolctl import threadpool_limits
    cfg = oracle.Config(batch=1, n_layers=1)
    cont = si.state_contents(1, 1, 4, 256, 1023, 1024, 256, seed=seed)
    st = oracle.state_from_arrays(cfg, {k: _np(v) for k, v in cont.items()}, pos=4096, bank_fill=1024, pend_fill=0)
    w, b = si.gate_params(1, 16, 256, seed)
    n_blocks = 16
    xs = [{k: _np(v) for k, v in si.prefill_inputs(1, 256, 4, 4, 256, seed=seed + j).items()} for j in range(n_blocks)]
    flops = prefill_flops(1, 1, 256, 20)[-1] * n_blocks   # blocks at steady state
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        for x in xs:
            oracle.prefill_block(st, 0, x["q"], x["k"], x["v"], x["cand_k"], x["cand_v"], x["cand_score"],
                                 w[0].numpy(), b[0].numpy())
        dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e9, "unit": "GFLOP/s", "cores": 1, "kind": "oracle",
            "sample": f"{n_blocks} blocks of 256 tokens x 1 sequence x 1 layer (ring and bank full, forced "
                      f"admits), FP64 numpy oracle, 1 thread; {dt:.1f} s", "cpu": host_cpu()}


def run_reference(args) -> None:
    """The reference arm: the CPU oracle as it stands, on this machine's host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # each step is a bounded sample of the batch-512 workload: one sequence x 8 layers
    import oracle
    import synth_inputs as si
    from threadpoolctl import threadpool_limits
    n_layers = 8
    cfg = oracle.Config(batch=1, n_layers=n_layers)
    n_src = 4   # sequences of the workload visited in turn
    states = []
    for sidx in range(n_src):
        cont = si.state_contents(n_layers, 1, 4, 256, 1023, 1024, 256, seed=sidx)
        c = si.workload_counters("batch", n_layers, 1, 4)
        c["pos"] += 64 * sidx
        c["pend_fill"] += 64 * sidx
        states.append(oracle.state_from_arrays(cfg, {k: _np(v) for k, v in cont.items()}, **c))
    w, b = si.gate_params(n_layers, 16, 256, 0)
    w, b = w.numpy(), b.numpy()
    pool = [[{k: _np(v) for k, v in si.decode_inputs(1, 4, 4, 256, seed=1000 * s + l).items()}
             for l in range(n_layers)] for s in range(16)]

    def step(i):
        st = states[i % n_src]
        for l in range(n_layers):
            x = pool[i % 16][l]
            oracle.decode_step(st, l, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                               x["cand_score"], w[l], b[l])
            oracle.admit(st, l)

    with threadpool_limits(limits=1):
        for i in range(args.warmup):
            step(i)
        t0 = time.perf_counter()
        for i in range(args.steps):
            step(args.warmup + i)
        dt = time.perf_counter() - t0
    value = args.steps / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "batch-512 decode, sampled: each step is one of the 512 sequences through "
                               "8 RMA layers (decode + admit), 4 KV groups x 4 q-heads, head_dim 256, "
                               "full ring and bank, staggered pending"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": "1 sequence x 8 layers per step (numpy FP64 oracle, 1 thread)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# block prefill workload
# ---------------------------------------------------------------------------

def prefill_flops(B: int, L: int, n: int, blocks: int, R: int = 1023, A: int = 1024, heads: int = 16,
                  D: int = 256) -> list:
    """Algorithmic FLOPs of each block call (one layer): 4 D per valid (query head, key) pair.

    Starting from an empty state, block j starts at s = n j with bank_fill =
    min(A, n j); query i sees min(s + i, R) + 1 window keys and bank_fill anchors.
    """
    out = []
    for j in range(blocks):
        s, bank = n * j, min(A, n * j)
        pairs = sum(min(s + i, R) + 1 + bank for i in range(n))
        out.append(B * heads * 4 * D * pairs)
    return out


def run_prefill(args) -> None:
    import torch
    from bounded_memory_attention_b200 import build
    build.build()
    import bounded_memory_attention_b200 as rma
    import synth_inputs as si
    device = torch.device("cuda", 0)
    B = args.batch or 8
    L, n, blocks = 8, 256, args.blocks
    cfg = rma.Config(batch=B, n_layers=L)
    st = rma.State(cfg, device=device)
    g = torch.Generator(device=device)
    g.manual_seed(0)
    for name in ("ring_k", "ring_v", "bank_k", "bank_v", "pend_k", "pend_v"):
        getattr(st, name).normal_(generator=g)
    st.bank_score.normal_(generator=g)
    st.pend_score.normal_(generator=g)
    w, bg = si.gate_params(L, 16, 256, 0, device=device)
    pool = [[si.prefill_inputs(B, n, 4, 4, 256, seed=100 * k + l, device=device) for l in range(L)] for k in range(4)]
    outs = torch.empty(B, n, 16, 256, dtype=torch.bfloat16, device=device)
    ws = st.workspace(n)
    stream = torch.cuda.current_stream(device)

    def block(j, strm):
        for l in range(L):
            x = pool[j % 4][l]
            rma.prefill_block(st, l, x["q"], x["k"], x["v"], x["cand_k"], x["cand_v"], x["cand_score"], w[l], bg[l],
                              outs, ws, stream=strm)

    # One CUDA graph per input set: the 8 layer calls of a block (the state's counters advance on the
    # device, so replaying a graph runs the next block).  --eager launches every call from Python.
    graphs = None
    if not args.eager:
        cs = torch.cuda.Stream(device)
        cs.wait_stream(stream)
        with torch.cuda.stream(cs):
            for j in range(4):
                block(j, cs)                  # warm-up outside the capture
        cs.synchronize()
        graphs = []
        for j in range(4):
            gph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gph, stream=cs):
                block(j, cs)
            graphs.append(gph)
        torch.cuda.synchronize(device)

    def run(j):
        if graphs is None:
            block(j, stream)
        else:
            graphs[j % 4].replay()

    for j in range(max(3, args.warmup)):
        run(j)
    st.counters.zero_()                       # the timed run starts from an empty state
    torch.cuda.synchronize(device)
    evs = [[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(blocks)]
    sampler = ClockSampler(None)
    sampler.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for j in range(blocks):
        evs[j][0].record(stream)
        run(j)
        evs[j][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    ms = t0.elapsed_time(t1)
    fl = prefill_flops(B, L, n, blocks)
    call_ms = [evs[j][0].elapsed_time(evs[j][1]) / L for j in range(blocks) for _ in range(L)]
    total_flops = sum(f * L for f in fl)
    with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
        pk = json.load(f)
    peak = float(pk["bf16_tflops_sustained"])
    achieved = total_flops / (sum(call_ms) / 1e3) / 1e12
    pf_traffic, pf_traffic_note = profiled_traffic("rma_prefill")
    line = {
        "metric": f"RMA block-prefill TFLOP/s (algorithmic), batch {B} x {L} layers x {blocks} blocks of {n}",
        "value": total_flops / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "tokens_per_s": B * n * blocks / (ms / 1e3),
        "n_gpus": 1, "steps": blocks, "ms_total": ms, "higher_is_better": True, "dtype": "bf16",
        "accumulate": "f32", "data": "synthetic",
        "config": {"workload": f"block prefill: {B} sequences x {L} RMA layers, {blocks} blocks of {n} queries "
                               "from an empty state; each block attends causally to the 1024-position window and "
                               "to the bank committed before it, then admits its 256 candidates",
                   "algorithmic_tflop": total_flops / 1e12,
                   "launch": "eager, one Python call per layer" if args.eager else
                             "each block's 8 layer calls replayed from a CUDA graph (inputs in fixed device buffers)",
                   "l2": f"inputs larger than L2: the {st.buffer.numel() / 1e6:.0f} MB state spans {L} layers and each call "
                         "reads another layer's ring and bank"},
        "clocks": clocks,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "traffic": pf_traffic, "traffic_note": pf_traffic_note,
                     "kernel": "rma_prefill_block: prefill_attn_kernel (about 80% of the call) + prefill_commit_kernel "
                               "+ prefill_admit_copy_kernel, timed together per call",
                     "call_ms_mean": sum(call_ms) / len(call_ms),
                     "call_ms_note": "per 8-layer block (CUDA events around each replay) / 8",
                     "peak_source": "measured bf16_tflops_sustained (MEASURED_PEAKS.json)"},
        "gpu_launches": blocks * L,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = all_and_one_core(lambda: cpu_oracle_prefill_allcores(n_blocks=16),
                                                cpu_oracle_prefill, "GFLOP/s")
    print(json.dumps(line), flush=True)


def admitted_counts(bank_score, pend_score):
    """How many candidates each group admits when every bank slot and every pending slot is
    filled: those among the first A of the A + P records ordered by score (descending), then
    committed before candidate, then slot (ascending).  bank_score [..., A] and pend_score
    [..., P] float32 without NaN -> int array [...].  Byte counting for the roofline only."""
    import numpy as np
    A, P = bank_score.shape[-1], pend_score.shape[-1]
    lead = bank_score.shape[:-1]
    sc = np.concatenate([bank_score.reshape(-1, A), pend_score.reshape(-1, P)], axis=1)
    cand = np.broadcast_to(np.r_[np.zeros(A, np.int8), np.ones(P, np.int8)], sc.shape)
    slot = np.broadcast_to(np.r_[np.arange(A), np.arange(P)], sc.shape)
    order = np.lexsort((slot, cand, -sc), axis=-1)       # -0.0 and +0.0 compare equal, as in the order
    return np.take_along_axis(cand, order[:, :A], axis=1).sum(axis=1).reshape(lead)


def cpu_oracle_admit(seed: int = 0, n_seq: int = 32, reps: int = 16) -> dict:
    """Time the oracle's admit on groups with every bank and pending slot filled (scores ~ N(0,1)),
    in algorithmic GB/s (one host thread); each repetition starts from a fresh copy of the state."""
    import oracle
    import synth_inputs as si
    from threadpoolctl import threadpool_limits
    cfg = oracle.Config(batch=n_seq, n_layers=1)
    cont = si.state_contents(1, n_seq, 4, 256, 1023, 1024, 256, seed=seed)
    st0 = oracle.state_from_arrays(cfg, {k: _np(v) for k, v in cont.items()}, pos=131_072, bank_fill=1024,
                                   pend_fill=256)
    n_adm = admitted_counts(st0.bank_score, st0.pend_score)
    nbytes = n_seq * 4 * ADMIT_SCORE_BYTES + ADMIT_ROW_BYTES * int(n_adm.sum())
    dt = 0.0
    with threadpool_limits(limits=1):
        for _ in range(reps):
            st = oracle.copy_state(st0)
            t0 = time.perf_counter()
            oracle.admit(st, 0)
            dt += time.perf_counter() - t0
    return {"value": reps * nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{reps} admits of {n_seq} sequences x 4 groups (one layer, every bank and pending "
                      f"slot filled), FP64/numpy oracle, 1 thread; {dt:.1f} s", "cpu": host_cpu()}


def run_admit(args) -> None:
    """The standalone admit of a batch whose sequences are in phase: every group's bank (1,024)
    and pending buffer (256) full, scores ~ N(0,1).  One step = rma_admit for each layer.  Before
    each step the bank scores and the counters are restored (untimed), so every step makes the
    same selection; the K/V rows the previous step copied stay, which changes no byte count."""
    import torch
    from bounded_memory_attention_b200 import build
    build.build()
    import bounded_memory_attention_b200 as rma
    device = torch.device("cuda", 0)
    B, L, G = args.batch or 512, args.layers or 8, 4
    st = rma.State(rma.Config(batch=B, n_layers=L), device=device)
    gen = torch.Generator(device=device)
    gen.manual_seed(0)
    for name in ("bank_k", "bank_v", "pend_k", "pend_v"):
        getattr(st, name).normal_(generator=gen)
    st.bank_score.normal_(generator=gen)
    st.pend_score.normal_(generator=gen)
    score0 = st.bank_score.clone()
    cnt0 = torch.zeros(L, B, G, 4, dtype=torch.int32, device=device)
    cnt0[..., 0], cnt0[..., 1], cnt0[..., 2] = 131_072, 1024, 256
    n_adm = admitted_counts(score0.cpu().numpy(), st.pend_score.cpu().numpy())   # [L, B, G]
    launch_bytes = [B * G * ADMIT_SCORE_BYTES + ADMIT_ROW_BYTES * int(n_adm[l].sum()) for l in range(L)]
    stream = torch.cuda.current_stream(device)

    def step(ev=None):
        st.bank_score.copy_(score0)
        st.counters.copy_(cnt0)
        for l in range(L):
            if ev is not None:
                ev[l][0].record(stream)
            rma.admit(st, l, stream=stream)          # runs where pending is full: every group
            if ev is not None:
                ev[l][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    # the bookkeeping above must describe what the kernel did: one changed score per admitted candidate
    changed = (st.bank_score != score0).sum(dim=-1).cpu().numpy()
    counts_agree = bool((changed == n_adm).all())
    K = args.steps
    evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(L)]
           for _ in range(K)]
    sampler = ClockSampler(None)
    sampler.start()
    for i in range(K):
        step(evs[i])
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    call_ms = [evs[i][l][0].elapsed_time(evs[i][l][1]) for i in range(K) for l in range(L)]
    admit_ms = sum(call_ms)
    total_bytes = K * sum(launch_bytes)
    achieved = total_bytes / (admit_ms / 1e3) / 1e9
    peak, peak_kind = peaks()
    # DRAM bytes of one full-size launch (2,048 groups), captured on this workload's default shape
    traffic, traffic_note = profiled_traffic("rma_admit") if B == 512 else (None, "captured at batch 512 only")
    line = {
        "metric": f"RMA admit GB/s (algorithmic), batch {B} x {L} layers, every bank and pending buffer full",
        "value": achieved, "unit": "GB/s", "n_gpus": 1, "steps": K, "warmup": args.warmup,
        "ms_per_step": admit_ms / K, "higher_is_better": True, "dtype": "u64", "data": "synthetic",
        "config": {"workload": f"admit: {B} sequences x {L} RMA layers x {G} KV groups, all in phase (banks full "
                               "with 1024 anchors, pending full with 256 candidates, scores ~ N(0,1)); one step = "
                               "rma_admit per layer",
                   "batch": B, "layers": L, "groups_per_launch": B * G,
                   "admitted_per_group_mean": float(n_adm.mean()),
                   "admitted_counts_match_kernel": counts_agree,
                   "l2": "inputs larger than L2: each launch reads its layer's pending K/V "
                         f"({B * G * 256 * 1024 / 1e9:.2f} GB) and writes into its bank "
                         f"({B * G * 1024 * 1024 / 1e9:.2f} GB); the {score0.numel() * 4 / 1e6:.0f} MB of bank "
                         "scores restored before each step (untimed) may sit in L2"},
        "clocks": clocks,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "traffic_note": traffic_note,
                     "kernel": "rma_admit (admit_kernel)", "kernel_ms": admit_ms,
                     "algorithmic_bytes_per_launch": sum(launch_bytes) / L,
                     "algorithmic_bytes_note": "5,120 B of scores per group + 2,052 B per admitted candidate "
                                               "(K and V rows read and written, its score written)",
                     "call_ms_mean": admit_ms / len(call_ms),
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured"
                     else "fallback 6.65 TB/s"},
        "gpu_launches": K * L,
    }
    if not args.no_cpu_baseline:
        try:
            line["cpu_baseline"] = cpu_oracle_admit()
        except Exception as ex:   # a report, never a reason to lose the bench line
            line["cpu_baseline"] = {"value": None, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                    "sample": f"failed: {ex}"}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the CUDA arm
# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1024)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--workload", default="batch", choices=["batch", "long", "ragged", "prefill", "admit"])
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--layers", type=int, default=None, help="admit workload: RMA layers (default 8)")
    ap.add_argument("--blocks", type=int, default=128, help="prefill workload: blocks of 256 tokens")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="prefill workload: launch every call from Python instead of replaying CUDA graphs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--splits", default=None,
                    help="decode workloads: ring,bank split counts (rma_set_decode_splits); default: the library's")
    ap.add_argument("--no-overlap", action="store_true",
                    help="decode workloads: leave rma_set_decode_overlap off (the library default)")
    ap.add_argument("--kv", default="bf16", choices=["bf16", "fp8"],
                    help="decode workloads: K/V storage (fp8: E4M3 codes with a per-row scale)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return
    if args.workload == "prefill":
        run_prefill(args)
        return
    if args.workload == "admit":
        if args.steps == 1024:       # the decode default; the admit workload takes fewer steps
            args.steps = 20
        run_admit(args)
        return

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    from bounded_memory_attention_b200 import build
    build.build()
    import bounded_memory_attention_b200 as rma
    import synth_inputs as si

    B = args.batch or {"batch": 512, "long": 1, "ragged": 512}[args.workload]
    L = 8
    kind = args.workload
    fp8 = args.kv == "fp8"
    cfg, st, w, b, pool = make_decode_workload(rma, torch, si, B, L, kind, seed=rank, device=device, fp8=fp8)
    if args.splits:   # before the workspace: its size follows the split shape
        rs, bs = (int(v) for v in args.splits.split(","))
        rma.set_decode_splits(st, rs, bs)
    ws = st.workspace(1)
    out = torch.empty(B, 16, 256, dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)
    # each launch of a step is another layer: with overlap on, it requests its first ring and bank
    # tiles while the previous layer's launch finishes (nothing else writes the state in this loop)
    rma.set_decode_overlap(st, not args.no_overlap)

    def step(i, ev=None, strm=None):
        strm = strm if strm is not None else stream
        for l in range(L):
            x = pool[i % 16][l]
            if ev is not None:
                ev[l][0].record(strm)
            rma.decode_step(st, l, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"], x["cand_score"],
                            w[l], b[l], out, ws, stream=strm)
            if ev is not None:
                ev[l][1].record(strm)

    # algorithmic bytes of every launch, from the counters the steps will see
    cnt0 = st.counters.cpu().numpy().astype("int64")
    fills = FillTracker(cnt0, fp8=fp8)
    step_bytes = fills.step_bytes

    # the long-context case is launch-latency bound: its 8 launches per step are replayed from
    # CUDA graphs (one per input set) instead of being issued one by one from Python
    graphs = None
    if kind == "long":
        cs = torch.cuda.Stream(device)
        cs.wait_stream(stream)
        with torch.cuda.stream(cs):
            step(0, strm=cs)
        cs.synchronize()
        graphs = []
        for sidx in range(16):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr, stream=cs):
                step(sidx, strm=cs)
            graphs.append(gr)
        torch.cuda.synchronize(device)
        st.counters.copy_(torch.from_numpy(cnt0).to(torch.int32))   # the captured steps ran nothing
        torch.cuda.synchronize(device)

    for i in range(args.warmup):
        if graphs is not None:
            graphs[i % 16].replay()
        else:
            step(i)
        step_bytes()
    K = args.steps
    evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(L)]
           for _ in range(K)]
    timed_bytes = []
    t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(device).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        uuid = None
    sampler = ClockSampler(uuid)
    sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    t0e.record(stream)
    for i in range(K):
        if graphs is not None:
            evs[i][0][0].record(stream)
            graphs[(args.warmup + i) % 16].replay()
            evs[i][0][1].record(stream)
        else:
            step(args.warmup + i, evs[i])
        timed_bytes.append(step_bytes())
    t1e.record(stream)
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = max_over_ranks(t0e.elapsed_time(t1e), world, device)
    ms_per_step = ms / K
    value = whole_job_rate(world, B * K, ms)

    # dominant kernel: rma_decode, per-launch duration from the events around each launch (for
    # the graph-replayed long-context steps: the step time over its 8 launches)
    latency = None
    if graphs is not None:
        step_ms = sorted(evs[i][0][0].elapsed_time(evs[i][0][1]) for i in range(K))
        dec_ms = sum(step_ms) / len(step_ms) / L
        latency = {"unit": "us per 8-layer step (CUDA graph replay)", "median": 1e3 * step_ms[len(step_ms) // 2],
                   "p99": 1e3 * step_ms[min(len(step_ms) - 1, int(0.99 * len(step_ms)))], "min": 1e3 * step_ms[0]}
    else:
        durs = [evs[i][l][0].elapsed_time(evs[i][l][1]) for i in range(K) for l in range(L)]
        dec_ms = sum(durs) / len(durs)
    alg_bytes = sum(timed_bytes) / (K * L)     # per launch, from the exact per-step fills
    dec_traffic, dec_traffic_note = (profiled_traffic("rma_decode_fp8" if fp8 else "rma_decode") if kind == "batch"
                                     else (None, "captured on the batch-512 workload only"))
    peak, peak_kind = peaks()

    # end to end through the public API: host (pinned) inputs in, host output out, every step
    e2e = None
    if not args.no_e2e:
        h2d, d2h = step_input_bytes(B, L)
        host_in = [[{k: v.cpu().pin_memory() for k, v in pool[s][l].items()} for l in range(L)] for s in range(4)]
        # two sets of device inputs and outputs, so that the copies of one step overlap the
        # kernels of the next: inputs go up on one copy stream, results come down on another
        host_out = [torch.empty(L, B, 16, 256, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        dev_in = [[{k: torch.empty_like(v, device=device) for k, v in host_in[0][l].items()} for l in range(L)]
                  for _ in range(2)]
        outs = [torch.empty(L, B, 16, 256, dtype=torch.bfloat16, device=device) for _ in range(2)]
        up, down = torch.cuda.Stream(device), torch.cuda.Stream(device)
        in_ready = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        read = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(n_steps):
            up.wait_stream(stream)
            down.wait_stream(stream)

            def h2d_of(i):
                k = i % 2
                if i >= 2:
                    up.wait_event(done[k])              # step i - 2 no longer reads these inputs
                with torch.cuda.stream(up):
                    for l in range(L):
                        for name, v in host_in[i % 4][l].items():
                            dev_in[k][l][name].copy_(v, non_blocking=True)
                in_ready[k].record(up)

            h2d_of(0)
            for i in range(n_steps):
                k = i % 2
                if i + 1 < n_steps:
                    h2d_of(i + 1)
                stream.wait_event(in_ready[k])
                if i >= 2:
                    stream.wait_event(read[k])          # step i - 2's results have come down
                for l in range(L):
                    x = dev_in[k][l]
                    rma.decode_step(st, l, x["q"], x["k_cur"], x["v_cur"], x["cand_k"], x["cand_v"],
                                    x["cand_score"], w[l], b[l], outs[k][l], ws, stream=stream)
                done[k].record(stream)
                down.wait_event(done[k])
                with torch.cuda.stream(down):
                    host_out[k].copy_(outs[k], non_blocking=True)
                read[k].record(down)
            stream.wait_stream(up)
            stream.wait_stream(down)

        Ke = max(16, K // 8)
        e2e_run(3)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        e2e_run(Ke)
        a1.record(stream)
        torch.cuda.synchronize(device)
        ems = max_over_ranks(a0.elapsed_time(a1), world, device)
        e2e = {"value": whole_job_rate(world, B * Ke, ems), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": Ke,
               "path": "pinned host inputs -> device copies (copy stream) -> rma_decode_step x 8 layers -> "
                       "pinned host outputs (second copy stream); two buffer sets, so the copies of one "
                       "step overlap the kernels of the next"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and kind == "batch" and not fp8:
        cpu = all_and_one_core(lambda: cpu_oracle_decode_allcores(n_steps=64),
                               lambda: cpu_oracle_decode(n_seq=8, n_layers=8, n_steps=12), UNIT)

    if rank == 0:
        line = {
            "metric": METRIC + (", FP8 E4M3 K/V storage" if fp8 else ""), "value": value, "unit": UNIT,
            "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8-e4m3 K/V (per-row power-of-two scale), bf16 Q/out" if fp8 else "bf16",
            "accumulate": "f32", "data": "synthetic",
            "config": {"workload": {"batch": "batch-512 decode: 512 sequences x 8 RMA layers, 4 KV groups x 4 "
                                             "q-heads, head_dim 256, rings full (1023), banks full (1024), pending "
                                             "staggered 0..255 (2 admits per layer per step)",
                                    "long": "long-context decode: 1 sequence x 8 RMA layers, pos 131072, full ring "
                                            "and bank, pending 0",
                                    "ragged": f"ragged decode: {B} sequences x 8 layers, ring fill U{{1..1023}}, "
                                              "bank fill U{0..1024}, pending U{0..255}, 16-level scores"}[kind],
                       "batch": B, "layers": L, "kv_storage": "fp8_e4m3" if fp8 else "bf16",
                       "decode_overlap": not args.no_overlap, "splits": args.splits or "library default",
                       "step": "8 x rma_decode_step (the admit runs inside the step that fills a pending buffer)",
                       "l2": "inputs larger than L2: the state is %.1f GB" % (st.buffer.numel() / 1e9),
                       "parallelism": f"replicas x{world} (no data-path collective)"},
            "gpu_launches": K * L,
            "clocks": clocks,
            "roofline": {"bound": "hbm",
                         "achieved": (alg_bytes / (dec_ms / 1e3) / 1e9) if alg_bytes else None,
                         "peak": peak, "unit": "GB/s",
                         "frac": (alg_bytes / (dec_ms / 1e3) / 1e9 / peak) if alg_bytes else None,
                         "traffic": dec_traffic, "traffic_note": dec_traffic_note,
                         "kernel": "rma_decode (decode_kernel)", "kernel_ms": dec_ms,
                         "algorithmic_bytes_per_launch": alg_bytes,
                         "algorithmic_bytes_note": ("ring min(pos, 1023) + bank_fill rows x " +
                                                    ("514 B (K and V codes + 2 exponents)" if fp8 else "1 KiB") +
                                                    " per group, plus q, out, current K/V and the ring write, from the "
                                                    "exact fills of every timed launch"),
                         "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured"
                         else "fallback 6.65 TB/s"},
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        if latency is not None:
            line["latency"] = latency
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
