#!/usr/bin/env python
"""Throughput of speculative-sampling verification on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step = one ``spec_verify`` call over one batch of the synthetic
quantized-self-draft workload (B=64 requests, k=8 drafts, V=151,936, bf16
logits, T=1) with its inputs already resident in HBM: the row-statistics
kernel over every used row, then the acceptance scan and the final draw.
Rank 0 prints one JSON line.

* value        verified draft positions/s over all ranks (sum of draft
               lengths per call x calls / max-over-ranks device time)
* e2e          the same metric through the host entry point
               (spec_verify_host): pinned host inputs copied in, results
               copied out, every step
* roofline     the row-statistics kernel: algorithmic bytes (every logit of
               every used row, read once) / its CUDA-event time, against the
               measured HBM copy bandwidth
* cpu_baseline the CPU oracle on the host cores (single thread), on a bounded
               sample of the same workload

With N > 1 (torchrun), every rank verifies its own batch (weak scaling); no
collective touches the data path, only the timing barrier and the max over
ranks.  ``--impl reference`` times the CPU oracle instead (rank 0 only).

``--host`` times the host-side components instead, on one CPU core and a
synthetic rollout history: per-request and batched n-gram drafting (lists
and one flat buffer), ranked candidates, suffix drafting, the prefetch
budget, and the fan-out prefetch pipeline's hit rate against its prediction.
"""
from __future__ import annotations

import argparse
import datetime
import itertools
import json
import math
import os
import statistics
import sys
import threading
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from speculative_decoding_verification_92_b200.workload import CONFIGS, config_seed, make_workload  # noqa: E402

METRIC = "verified draft positions/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
UNIT = "positions/s"
FALLBACK_HBM_GBS = 6650.0
MAX_REQUESTS_PER_STATS_LAUNCH = 4096     # mirrors the library's launch split
MAX_REQUESTS_PER_DRAW_LAUNCH = 65535
TRAFFIC_FILE = ROOT / "profiles" / "row_stats_traffic.json"

NVML_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=2, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--stats-kernel", default="auto", choices=["auto", "tma", "vec16", "scalar"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--greedy", action="store_true", help="time the greedy (prefix-match) form instead")
    ap.add_argument("--event-every", type=int, default=16,
                    help="bracket the row-statistics kernel with events on every N-th timed step")
    ap.add_argument("--host", action="store_true",
                    help="time the host-side drafters and prefetch budget instead (CPU only)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# workload bookkeeping


def rank_seed(cfg: int, rank: int) -> int:
    """Each rank verifies its own batch (weak scaling): rank r draws the
    workload from seed config_seed(cfg) + 7919 * r."""
    return config_seed(cfg) + 7919 * rank


def make_rank_workload(cfg: int, rank: int):
    params = dict(CONFIGS[cfg])
    return make_workload(seed=rank_seed(cfg, rank), **params)


def max_over_ranks(value: float, device=None) -> float:
    """The largest of every rank's value (timing only; no data-path
    collective).  Single process: the value itself."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(n_ranks: int, positions_per_step: int, steps: int, t_max_ms: float) -> float:
    """Whole-job verified draft positions/s: every rank verified
    positions_per_step positions per step; the job took the slowest rank's
    time."""
    return n_ranks * positions_per_step * steps / (t_max_ms / 1e3)


def stats_pass_bytes(w, greedy=False) -> int:
    """Algorithmic bytes of one call: every logit of every row the rule must
    read (target rows 0..L_b, draft rows 0..L_b-1), once."""
    L = w.draft_lens.astype(np.int64)
    rows = int((L + 1).sum())
    if w.draft is not None and not greedy:
        rows += int(L.sum())
    return rows * w.V * w.esize


def input_bytes(w, greedy=False) -> int:
    n = w.target.nbytes + w.tokens.nbytes
    if w.draft is not None and not greedy:
        n += w.draft.nbytes
    if w.lens is not None:
        n += w.lens.nbytes
    if not greedy:
        n += w.uniforms.nbytes
    return int(n)


def workload_desc(w, cfg) -> dict:
    return {
        "workload": f"{w.name}: B={w.B} k={w.k_max} V={w.V} {w.dtype} T={w.temperature}"
                    + (" one-hot q (no draft logits)" if w.draft is None else " draft logits")
                    + (" L in {0,4,12}" if w.lens is not None else ""),
        "config_id": cfg, "B": w.B, "k_max": w.k_max, "V": w.V, "input_dtype": w.dtype,
        "temperature": w.temperature, "draft": "ids" if w.draft is None else "logits",
        "positions_per_step": w.positions, "seed": config_seed(cfg),
    }


def measured_peak():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            d = json.loads(p.read_text())
            return float(d["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def committed_traffic(kernel_variant: str, cfg: int):
    """Per-launch DRAM bytes of the row-statistics kernel from the committed
    ncu summary, only if it was taken on the current kernel sources."""
    if not TRAFFIC_FILE.exists():
        return None
    try:
        from speculative_decoding_verification_92_b200 import build as _b
        d = json.loads(TRAFFIC_FILE.read_text())
        if d.get("source_hash") != _b.kernel_source_hash():
            return None
        e = d.get("per_config", {}).get(str(cfg), {}).get(kernel_variant)
        return None if e is None else float(e["dram_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nvml = pynvml
            props = torch.cuda.get_device_properties(device_index)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report what we have
            log(f"clock sampling unavailable: {e}")
        self.period = period_s
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                try:
                    r = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    r = n.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.reasons |= int(r)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.ok:
            self.thread.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [v for k, v in NVML_REASONS.items() if self.reasons & k]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# CPU oracle timing


def time_oracle(w, n_requests: int, seconds: float, greedy=False, min_reps=1):
    """Run the oracle on the first n_requests of the batch until `seconds`
    have passed (at least min_reps times); returns (positions/s, reps,
    positions per rep, seconds)."""
    from oracle import default
    orc = default()
    sl = slice(0, n_requests)
    lens = None if w.lens is None else w.lens[sl]
    u = w.uniforms[sl].astype(np.float64)
    positions = int(w.draft_lens[sl].sum())
    reps, t0 = 0, time.perf_counter()
    while True:
        orc.verify(w.target[sl], None if (greedy or w.draft is None) else w.draft[sl], w.tokens[sl], lens,
                   None if greedy else u, w.temperature, greedy, V=w.V)
        reps += 1
        el = time.perf_counter() - t0
        if reps >= min_reps and el >= seconds:
            break
    return positions * reps / el, reps, positions, el


# ---------------------------------------------------------------------------


def run_reference(args):
    """CPU oracle arm: rank 0 alone; every step verifies a bounded sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = make_rank_workload(args.config, 0)
    from oracle import default
    orc = default()
    # calibrate the per-request cost, then size the per-step sample so that
    # warm-up + steps stay within about two minutes
    t0 = time.perf_counter()
    orc.verify(w.target[:1], None if w.draft is None else w.draft[:1], w.tokens[:1],
               None if w.lens is None else w.lens[:1], w.uniforms[:1].astype(np.float64), w.temperature,
               args.greedy, V=w.V)
    per_req = max(time.perf_counter() - t0, 1e-4)
    budget = 120.0 / max(1, args.steps + args.warmup)
    n_req = int(max(1, min(w.B, budget // per_req)))
    sl = slice(0, n_req)
    lens = None if w.lens is None else w.lens[sl]
    u = w.uniforms[sl].astype(np.float64)
    draft = None if (w.draft is None or args.greedy) else w.draft[sl]
    positions = int(w.draft_lens[sl].sum())
    for _ in range(args.warmup):
        orc.verify(w.target[sl], draft, w.tokens[sl], lens, u, w.temperature, args.greedy, V=w.V)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        orc.verify(w.target[sl], draft, w.tokens[sl], lens, u, w.temperature, args.greedy, V=w.V)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = positions * args.steps / total
    sample = f"first {n_req} of {w.B} requests ({positions} draft positions) per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_desc(w, args.config),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_host(args):
    """Host-side components on a synthetic RL rollout history: 64 prompts x 5
    rollouts per step over W = 4 steps (the NgramRL setup), each rollout a
    copy of the prompt's previous one with 10% of its tokens replaced.
    Times draft lookups (k = 16) and ranked candidates (f = 16) of the C++
    n-gram and suffix drafters, and the prefetch allocation; the plain-Python
    oracle is timed on a bounded sample of the same lookups."""
    import numpy as np

    from speculative_decoding_verification_92_b200 import host
    from oracle import host_policy as ho

    rng = np.random.default_rng(92)
    P, R, T, W, V = 64, 5, 1024, 4, 151936
    base = [rng.integers(0, V, T).astype(np.int32) for _ in range(P)]
    ng, sx, o_ng = host.NgramDrafter(6, W), host.SuffixDrafter(8), ho.NgramOracle(6, W)
    t0 = time.perf_counter()
    for step in range(W):
        ng.begin_step()
        o_ng.begin_step()
        for p in range(P):
            for r in range(R):
                roll = base[p].copy()
                m = rng.random(T) < 0.1
                roll[m] = rng.integers(0, V, int(m.sum()))
                ng.add(p, roll)
                o_ng.add(p, roll)
                if step == W - 1:
                    sx.append(p, r, roll)
                base[p] = roll
    build_s = time.perf_counter() - t0
    queries = [(int(rng.integers(0, P)), int(rng.integers(8, T))) for _ in range(20000)]
    ctxs = [base[p][max(0, q - 32):q] for p, q in queries]

    def rate(fn, items, budget_s):
        n, t0 = 0, time.perf_counter()
        for it in items:
            fn(*it)
            n += 1
            if time.perf_counter() - t0 > budget_s:
                break
        return n / (time.perf_counter() - t0), n

    items = [(p, c) for (p, _), c in zip(queries, ctxs)]
    ng_rate, _ = rate(lambda p, c: ng.draft(p, c, 16), items, 5.0)
    ng_cand, _ = rate(lambda p, c: ng.candidates(p, c, 16), items, 5.0)
    sx_rate, _ = rate(lambda p, c: sx.draft(p, c, 16), items, 5.0)
    o_rate, o_n = rate(lambda p, c: o_ng.draft(p, list(c), 16), items, args.cpu_seconds)
    pf = host.PrefetchBudget(16, 16, 256)
    for _ in range(256):
        pf.observe(int(rng.integers(0, 17)), int(rng.integers(-1, 16)))
    pf_rate, _ = rate(lambda b: pf.allocate(b), [(16,)] * 200000, 2.0)
    accepted = []
    for p, c in items[:2000]:
        d = ng.draft(p, c, 16)
        accepted.append(len(d))

    # batched drafting of whole verification batches (B = 128 requests per
    # call, the n-gram workload's batch) straight into draft_tokens / draft_lens
    Bq = 128
    batches = [([p for p, _ in items[i:i + Bq]], [c for _, c in items[i:i + Bq]])
               for i in range(0, len(items) - Bq + 1, Bq)]

    def batch_rate(threads):
        n, t0 = 0, time.perf_counter()
        for pids, cs in itertools.cycle(batches):
            ng.draft_batch(pids, cs, 16, n_threads=threads)
            n += Bq
            if time.perf_counter() - t0 > 3.0:
                break
        return n / (time.perf_counter() - t0)
    batch_1, batch_all = batch_rate(1), batch_rate(0)
    # the same batches with their contexts already in one buffer
    flat_batches = []
    for pids, cs in batches:
        off = np.zeros(len(cs) + 1, np.int64)
        np.cumsum([len(c) for c in cs], out=off[1:])
        flat_batches.append((pids, np.concatenate(cs).astype(np.int32), off))
    n, t0 = 0, time.perf_counter()
    for pids, flat, off in itertools.cycle(flat_batches):
        ng.draft_batch_flat(pids, flat, off, 16, n_threads=1)
        n += Bq
        if time.perf_counter() - t0 > 3.0:
            break
    batch_flat = n / (time.perf_counter() - t0)

    # fan-out prefetch: the whole pipeline (budget, drafting ahead, serving
    # with a synchronous fallback) along fresh rollouts of the same prompts,
    # verified by prefix match against them
    fp = host.FanoutPrefetcher(ng, k=16, budget=16, fmax=16, window=256)
    preds, t_prep, n_steps = [], 0.0, 0
    for p in range(8):
        text = base[p].copy()
        m = rng.random(T) < 0.1
        text[m] = rng.integers(0, V, int(m.sum()))
        text = [int(x) for x in text]
        pos = 8
        while pos < T - 18:
            ctx = text[:pos]
            d = [int(x) for x in ng.draft(p, ctx, 16)]
            t0 = time.perf_counter()
            preds.append(fp.prepare(n_steps, p, ctx, d))
            t_prep += time.perf_counter() - t0
            j = 0
            while j < len(d) and d[j] == text[pos + j]:
                j += 1
            fp.next_draft(n_steps, j, text[pos + j])
            n_steps += 1
            pos += j + 1
    fanout = {"steps": n_steps, "hit_rate": fp.hits / max(n_steps, 1),
              "predicted_hit_rate": float(np.mean(preds)) if preds else 0.0,
              "prepare_us": 1e6 * t_prep / max(n_steps, 1)}
    line = {
        "metric": "host n-gram draft lookups/s (k=16), 1 core", "value": ng_rate, "unit": "lookups/s",
        "data": "synthetic", "config": {"workload": f"{P} prompts x {R} rollouts x {T} tokens, W={W} steps, "
                                                    "10% token changes per rollout", "max_n": 6, "k": 16},
        "ngram_candidates_per_s": ng_cand, "suffix_draft_per_s": sx_rate, "prefetch_allocations_per_s": pf_rate,
        "ngram_batch_drafts_per_s": {"batch": Bq, "threads_1": batch_1, "threads_all": batch_all,
                                     "flat_buffer_threads_1": batch_flat, "hardware_threads": os.cpu_count()},
        "fanout_prefetch": fanout,
        "table_build_s": build_s, "retained_tokens": ng.tokens, "mean_draft_len": float(np.mean(accepted)),
        "cpu_baseline": {"value": o_rate, "unit": "lookups/s", "cores": 1, "kind": "oracle",
                         "sample": f"{o_n} n-gram draft lookups with the plain-Python oracle"},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.host:
        return run_host(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours_impl(args)


def run_ours_impl(args):
    import torch
    import torch.distributed as dist

    import speculative_decoding_verification_92_b200 as sv

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        log(f"--gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE")
    n = world
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if n > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if n > 1:
            dist.barrier()

    sv.library()  # build / load before timing anything
    w = make_rank_workload(args.config, rank)
    greedy = bool(args.greedy)
    kernel = {"auto": sv.StatsKernel.AUTO, "tma": sv.StatsKernel.TMA, "vec16": sv.StatsKernel.VEC16,
              "scalar": sv.StatsKernel.SCALAR}[args.stats_kernel]

    def dev_tensor(a, bf16=False):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if bf16:
            t = t.view(torch.bfloat16)
        return t.to(dev)

    is_bf16 = w.dtype == "bf16"
    target = dev_tensor(w.target, is_bf16)
    draft = None if (w.draft is None or greedy) else dev_tensor(w.draft, is_bf16)
    tokens = dev_tensor(w.tokens)
    lens = None if w.lens is None else dev_tensor(w.lens)
    uniforms = None if greedy else dev_tensor(w.uniforms)
    out = (torch.empty(w.B, dtype=torch.int32, device=dev),
           torch.empty(w.B, w.k_max + 1, dtype=torch.int32, device=dev))
    ws = torch.empty(max(sv.workspace_bytes(w.B, w.k_max, w.V, sv.BF16 if is_bf16 else sv.F32), 256),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    in_bytes = input_bytes(w, greedy)
    flush_buf = None
    if in_bytes < 2 * l2:
        flush_buf = torch.empty(4 * l2 // 4, dtype=torch.int32, device=dev)
    l2_note = (f"inputs {in_bytes / 1e6:.1f} MB > 2 x L2 ({l2 / 2**20:.0f} MiB): no flush" if flush_buf is None
               else f"inputs {in_bytes / 1e6:.1f} MB < 2 x L2: L2 flushed (write {flush_buf.numel() * 4 / 2**20:.0f}"
                    f" MiB) before every step, outside each step's events")

    def step(events=None):
        sv.spec_verify(target, draft, tokens, lens, uniforms, w.temperature, greedy, V=w.V, out=out,
                       workspace=ws, stream=stream, stats_kernel=kernel, events=events)

    def new_event():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        return e

    K, W = args.steps, args.warmup
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    # Events cost a few microseconds each on the stream, so only every
    # EVENT_EVERY-th step brackets the row-statistics kernel; steps are timed
    # individually only when the L2 is flushed between them.
    every = max(1, args.event_every)
    k1_ev = {i: (new_event(), new_event()) for i in range(0, K, every)}
    step_ev = [(new_event(), new_event()) for _ in range(K)] if flush_buf is not None else None
    g0, g1 = new_event(), new_event()
    torch.cuda.synchronize()

    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        g0.record(stream)
        for i in range(K):
            if flush_buf is not None:
                flush_buf.fill_(i)
                step_ev[i][0].record(stream)
            step(events=k1_ev.get(i))
            if flush_buf is not None:
                step_ev[i][1].record(stream)
        g1.record(stream)
        torch.cuda.synchronize()
    barrier()

    k1_ms = [a.elapsed_time(b) for a, b in k1_ev.values()]
    region_ms = g0.elapsed_time(g1)
    step_ms = [a.elapsed_time(b) for a, b in step_ev] if step_ev is not None else [region_ms / K]
    t_rank = sum(step_ms) if flush_buf is not None else region_ms
    t_max = max_over_ranks(t_rank, dev)
    positions = w.positions
    value = aggregate_value(n, positions, K, t_max)
    ms_per_step = t_max / K

    # parity spot check of the timed outputs (host side, cheap): accept lengths in range
    g_len = out[0].cpu().numpy()
    assert np.all((g_len >= 0) & (g_len <= w.draft_lens)), "timed run produced invalid outputs"
    accept_rate = float(g_len.sum() / max(1, positions))

    # ---------------- end to end through the host entry point ----------------
    e2e = None
    if args.e2e_steps > 0:
        pin = lambda a, bf=False: (torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16) if bf
                                   else torch.from_numpy(np.ascontiguousarray(a))).pin_memory()
        h_target = pin(w.target, is_bf16)
        h_draft = None if draft is None else pin(w.draft, is_bf16)
        h_tokens, h_lens = pin(w.tokens), (None if w.lens is None else pin(w.lens))
        h_u = None if greedy else pin(w.uniforms)
        h_out = (torch.empty(w.B, dtype=torch.int32).pin_memory(),
                 torch.empty(w.B, w.k_max + 1, dtype=torch.int32).pin_memory())
        staging = torch.empty(sv.host_staging_bytes(w.B, w.k_max, w.V, sv.BF16 if is_bf16 else sv.F32,
                                                    has_draft=h_draft is not None, has_lens=h_lens is not None),
                              dtype=torch.uint8, device=dev)

        def e2e_step():
            sv.spec_verify_host(h_target, h_draft, h_tokens, h_lens, h_u, w.temperature, greedy, V=w.V,
                                out=h_out, staging=staging, workspace=ws, stream=stream)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        ev = [(new_event(), new_event()) for _ in range(args.e2e_steps)]
        barrier()
        torch.cuda.synchronize()
        for i in range(args.e2e_steps):
            ev[i][0].record(stream)
            e2e_step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev)
        assert np.array_equal(h_out[0].numpy(), g_len), "host entry point disagrees with device entry point"
        e2e = {"value": aggregate_value(n, positions, args.e2e_steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": int(h_out[0].nbytes + h_out[1].nbytes),
               "steps": args.e2e_steps, "ms_per_step": e2e_ms / args.e2e_steps}

    # ---------------- roofline of the row-statistics kernel ----------------
    peak, peak_kind = measured_peak()
    alg = stats_pass_bytes(w, greedy)
    k1_mean = statistics.fmean(k1_ms)
    achieved = alg / (k1_mean / 1e3) / 1e9
    variant = "tma" if args.stats_kernel == "auto" else args.stats_kernel
    traffic = committed_traffic(variant, args.config)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": traffic, "peak_kind": f"{peak_kind} (copy bandwidth, MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6650 GB/s",
                "kernel": f"row_stats ({variant})", "algorithmic_bytes_per_launch": alg,
                "kernel_ms": k1_mean, "kernel_ms_p10": float(np.percentile(k1_ms, 10)),
                "whole_step_gbs": alg / (ms_per_step / 1e3) / 1e9}

    launches_per_call = math.ceil(w.B / MAX_REQUESTS_PER_STATS_LAUNCH) + math.ceil(w.B / MAX_REQUESTS_PER_DRAW_LAUNCH)

    # ---------------- CPU oracle baseline (rank 0, N = 1) ----------------
    cpu = None
    if rank == 0 and n == 1 and not args.no_cpu_baseline:
        v, reps, pos, el = time_oracle(w, w.B, args.cpu_seconds, greedy)
        cpu = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"whole batch ({w.B} requests, {pos} draft positions) x {reps} passes, {el:.1f} s,"
                         f" single-threaded C, fp64"}

    if rank == 0:
        cfgd = workload_desc(w, args.config)
        cfgd.update({"parallelism": f"replicas{n}" if n > 1 else "single",
                     "sharding": "each rank verifies its own batch; no data-path collective",
                     "l2": l2_note, "stats_kernel": variant, "greedy": greedy})
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": n, "steps": K, "warmup": W,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic", "config": cfgd,
            "e2e": e2e, "gpu_launches": K * launches_per_call, "roofline": roofline,
            "cpu_baseline": cpu, "clocks": clocks.summary(),
            "hbm_gbs": alg / (ms_per_step / 1e3) / 1e9,
            "accept_rate": accept_rate, "mean_accept_len": float(g_len.mean()),
            "timing": {"region_ms": region_ms, "k1_event_samples": len(k1_ms), "k1_event_every": every,
                       "k1_ms_median": float(np.median(k1_ms))},
        }
        print(json.dumps(line), flush=True)
    if n > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
