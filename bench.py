#!/usr/bin/env python
"""Throughput of speculative-sampling verification on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

One step = one ``spec_verify`` call over one batch of a synthetic workload
with its inputs already resident in HBM: the row-statistics kernel over every
used row, then the acceptance scan and the final draw.  The default workload
is the largest single-GPU one, the length-aware-budgets batch (B=256,
k_max=12, per-request draft lengths in {0, 4, 12}, V=128,256, fp32 logits,
T=1, about 1 GB of logits read per step).  Rank 0 prints one JSON line.

* value        verified draft positions/s over all ranks (sum of draft
               lengths per call x calls / max-over-ranks device time)
* e2e          the same metric through the host entry point
               (spec_verify_host): pinned host inputs copied in, results
               copied out, every step
* roofline     the row-statistics kernel: algorithmic bytes (every logit of
               every used row, read once) / its mean CUDA-event time over a
               separate pass of at least 10 launches, against the measured
               HBM copy bandwidth; the whole step's bandwidth beside it
* per_config   the same figures for the four other workloads (1 GPU), each
               with a parity spot check (outputs well formed, host entry
               point equal to the device entry point)
* cpu_baseline the CPU oracle on every hardware thread of the host (and
               single-threaded on a sample), on the same workload

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
NOMINAL_HBM_GBS = 8000.0                 # B200 HBM3e, vendor figure (context only)
MAX_REQUESTS_PER_STATS_LAUNCH = 4096     # mirrors the library's launch split
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
    ap.add_argument("--config", type=int, default=5, choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--stats-kernel", default="auto", choices=["auto", "tma", "vec16", "scalar"])
    ap.add_argument("--draw-path", default="auto", choices=["auto", "queue", "cluster"],
                    help="how sampling calls make their final draws (the library's AUTO by default)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--greedy", action="store_true", help="time the greedy (prefix-match) form instead")
    ap.add_argument("--k1-samples", type=int, default=50,
                    help="launches of the row-statistics kernel timed with events (at least 10)")
    ap.add_argument("--per-config-steps", type=int, default=200,
                    help="timed steps of each other workload in the per_config block")
    ap.add_argument("--no-per-config", action="store_true", help="time the chosen workload only")
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


def host_copy_bytes(w, greedy=False) -> int:
    """Bytes spec_verify_host copies to the device per call: the logit rows
    the method reads (target rows 0..L_b, draft rows 0..L_b-1; every row when
    no draft_lens are given), the ids, lengths and uniforms."""
    if w.lens is None:
        return input_bytes(w, greedy)
    row = w.target.shape[2] * w.target.itemsize
    L = np.clip(w.lens.astype(np.int64), 0, w.k_max)
    n = int((L + 1).sum()) * row + w.tokens.nbytes + w.lens.nbytes
    if w.draft is not None and not greedy:
        n += int(L.sum()) * row
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
        if d.get("source_hash") != _b.row_stats_source_hash():
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


def _request_slices(w, n_parts: int):
    """Contiguous request ranges of about equal row counts (the oracle's work
    is proportional to the rows it reads)."""
    rows = (w.draft_lens.astype(np.int64) + 1) * (2 if w.draft is not None else 1)
    cum = np.concatenate([[0], np.cumsum(rows)])
    cuts = [int(np.searchsorted(cum, cum[-1] * i / n_parts)) for i in range(n_parts + 1)]
    cuts[0], cuts[-1] = 0, w.B
    return [slice(a, b) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]


def _oracle_call(orc, w, sl, greedy):
    lens = None if w.lens is None else w.lens[sl]
    orc.verify(w.target[sl], None if (greedy or w.draft is None) else w.draft[sl], w.tokens[sl], lens,
               None if greedy else w.uniforms[sl].astype(np.float64), w.temperature, greedy, V=w.V)


def time_oracle(w, seconds: float, greedy=False, threads: int = 1, n_requests: int | None = None):
    """Run the oracle over the first n_requests (default all) of the batch,
    split into `threads` contiguous request ranges verified concurrently (the
    oracle's C entry point releases the GIL; each request is still verified
    sequentially), until `seconds` have passed.  Returns (positions/s, passes,
    positions per pass, seconds, threads used)."""
    from concurrent.futures import ThreadPoolExecutor
    from oracle import default
    orc = default()
    n = w.B if n_requests is None else max(1, min(w.B, n_requests))
    sub = w if n == w.B else _sub_workload(w, n)
    slices = _request_slices(sub, max(1, threads))
    positions = int(sub.draft_lens.sum())
    passes, t0 = 0, time.perf_counter()
    with ThreadPoolExecutor(max_workers=len(slices)) as ex:
        while True:
            list(ex.map(lambda sl: _oracle_call(orc, sub, sl, greedy), slices))
            passes += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
    return positions * passes / el, passes, positions, el, len(slices)


def _sub_workload(w, n):
    """The first n requests of a workload (views, no copies)."""
    import dataclasses
    return dataclasses.replace(w, B=n, target=w.target[:n], draft=None if w.draft is None else w.draft[:n],
                               tokens=w.tokens[:n], lens=None if w.lens is None else w.lens[:n],
                               uniforms=w.uniforms[:n], favoured=None if w.favoured is None else w.favoured[:n])


def oracle_baseline(w, seconds: float, greedy=False):
    """The oracle on the host's cores: single-threaded on a sample of the
    batch, then on the whole batch with one thread per hardware thread."""
    cores = os.cpu_count() or 1
    per_req = stats_pass_bytes(w, greedy) / max(1, w.B)
    n1 = int(max(1, min(w.B, 2e9 / max(per_req, 1))))        # ~1-2 s of single-threaded work per pass
    v1, p1, pos1, el1, _ = time_oracle(w, seconds / 2, greedy, threads=1, n_requests=n1)
    vn, pn, posn, eln, used = time_oracle(w, seconds / 2, greedy, threads=cores)
    return {"value": vn, "unit": UNIT, "cores": used, "host_cores": cores, "kind": "oracle",
            "single_thread_value": v1,
            "sample": f"all {w.B} requests ({posn} draft positions) x {pn} passes in {eln:.1f} s on {used} threads "
                      f"(contiguous request ranges, one per hardware thread); single thread: first {n1} requests "
                      f"({pos1} positions) x {p1} passes in {el1:.1f} s; plain C, fp64"}


# ---------------------------------------------------------------------------


def run_reference(args):
    """CPU oracle arm: rank 0 alone, on every hardware thread of the host;
    every step verifies a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = make_rank_workload(args.config, 0)
    cores = os.cpu_count() or 1
    # calibrate the per-request cost, then size the per-step sample so that
    # warm-up + steps stay within about two minutes
    t0 = time.perf_counter()
    _oracle_call(__import__("oracle").default(), w, slice(0, 1), args.greedy)
    per_req = max(time.perf_counter() - t0, 1e-4)
    budget = 120.0 / max(1, args.steps + args.warmup)
    n_req = int(max(1, min(w.B, cores * budget // per_req)))
    sub = w if n_req == w.B else _sub_workload(w, n_req)
    for _ in range(args.warmup):
        time_oracle(sub, 0.0, args.greedy, threads=cores)
    times, positions, used = [], int(sub.draft_lens.sum()), 1
    for _ in range(args.steps):
        v, passes, positions, el, used = time_oracle(sub, 0.0, args.greedy, threads=cores)
        times.append(el / passes)
    total = sum(times)
    value = positions * args.steps / total
    sample = (f"first {n_req} of {w.B} requests ({positions} draft positions) per step, "
              f"on {used} threads (one contiguous request range each)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_desc(w, args.config),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "host_cores": cores, "kind": "oracle",
                         "sample": sample},
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


class DeviceWorkload:
    """One workload resident on the device, with its output buffers and
    workspace, and the call that verifies it.

    Workloads smaller than twice the L2 cache are held in N device copies and
    step i verifies copy i mod N, with N chosen so that at least 2 x L2 of
    other inputs are read between two uses of one copy: every step reads its
    logits from HBM, as a fresh batch would be, and no cache flush (whose
    dirty lines would be written back inside the timed step) is needed."""

    def __init__(self, sv, torch, dev, stream, w, greedy, kernel, draw_path=0):
        self.sv, self.torch, self.dev, self.stream, self.w = sv, torch, dev, stream, w
        self.greedy, self.kernel, self.draw_path = greedy, kernel, draw_path
        self.is_bf16 = w.dtype == "bf16"
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.in_bytes = input_bytes(w, greedy)
        self.copies = 1 if self.in_bytes >= 2 * l2 else -(-2 * l2 // self.in_bytes) + 1

        def t(a, bf=False):
            x = torch.from_numpy(np.ascontiguousarray(a))
            if bf:
                x = x.view(torch.bfloat16)
            x = x.to(dev)
            if self.copies == 1:
                return [x]
            stacked = x.unsqueeze(0).repeat(self.copies, *([1] * x.dim())).contiguous()
            return [stacked[i] for i in range(self.copies)]

        self.target = t(w.target, self.is_bf16)
        self.draft = None if (w.draft is None or greedy) else t(w.draft, self.is_bf16)
        self.tokens = t(w.tokens)
        self.lens = None if w.lens is None else t(w.lens)
        self.uniforms = None if greedy else t(w.uniforms)
        self.out = (torch.empty(w.B, dtype=torch.int32, device=dev),
                    torch.empty(w.B, w.k_max + 1, dtype=torch.int32, device=dev))
        self.ws = torch.empty(max(sv.workspace_bytes(w.B, w.k_max, w.V, sv.BF16 if self.is_bf16 else sv.F32), 256),
                              dtype=torch.uint8, device=dev)
        self.l2_note = (f"inputs {self.in_bytes / 1e6:.1f} MB > 2 x L2 ({l2 / 2**20:.0f} MiB): no flush"
                        if self.copies == 1 else
                        f"inputs {self.in_bytes / 1e6:.1f} MB < 2 x L2 ({l2 / 2**20:.0f} MiB): {self.copies} device "
                        f"copies, step i reads copy i mod {self.copies} "
                        f"({(self.copies - 1) * self.in_bytes / 1e6:.0f} MB of other inputs between two reads of one "
                        f"copy), no flush")
        self._i = 0

    def step(self, events=None, copy=None):
        w = self.w
        c = self._i % self.copies if copy is None else copy
        self._i += 1
        pick = lambda x: None if x is None else x[c]
        self.sv.spec_verify(pick(self.target), pick(self.draft), pick(self.tokens), pick(self.lens),
                            pick(self.uniforms), w.temperature, self.greedy, V=w.V, out=self.out, workspace=self.ws,
                            stream=self.stream, stats_kernel=self.kernel, events=events, draw_path=self.draw_path)

    def event(self):
        e = self.torch.cuda.Event(enable_timing=True)
        e.record(self.stream)
        return e

    def time_steps(self, steps, warmup, barrier=lambda: None):
        """Time `steps` calls back to back between two events; returns the
        device ms of the timed calls."""
        torch = self.torch
        for _ in range(warmup):
            self.step()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        g0 = self.event()
        for _ in range(steps):
            self.step()
        g1 = self.event()
        torch.cuda.synchronize()
        barrier()
        return g0.elapsed_time(g1)

    def time_k1(self, samples):
        """The row-statistics kernel alone: `samples` calls, each with events
        recorded just before and after that kernel on the launching stream
        (a separate pass, so the events do not disturb the timed steps).
        Returns the per-launch times in ms."""
        torch = self.torch
        ev = []
        for _ in range(samples):
            # recorded once here so that torch creates the events; the
            # library records them again around the row-statistics kernel
            a, b = self.event(), self.event()
            self.step(events=(a, b))
            ev.append((a, b))
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    def host_check(self):
        """Parity spot check of the device outputs: every accept length lies
        in [0, L_b], the accepted prefix repeats the drafts, the emitted
        token is a vocabulary id and -1 fills the rest; and the host entry
        point (spec_verify_host, host buffers) returns the same outputs."""
        torch, w = self.torch, self.w
        self.step(copy=0)
        torch.cuda.synchronize()
        g_len = self.out[0].cpu().numpy()
        g_tok = self.out[1].cpu().numpy()
        L = w.draft_lens
        ok = bool(np.all((g_len >= 0) & (g_len <= L)))
        for b in range(w.B) if ok else ():
            j = int(g_len[b])
            ok &= bool(np.array_equal(g_tok[b, :j], w.tokens[b, :j]) and 0 <= g_tok[b, j] < w.V
                       and np.all(g_tok[b, j + 1:] == -1))
        h = self.host_buffers()
        self.sv.spec_verify_host(*h["inputs"], w.temperature, self.greedy, V=w.V, out=h["out"],
                                 staging=h["staging"], workspace=self.ws, stream=self.stream)
        torch.cuda.synchronize()
        same = bool(np.array_equal(h["out"][0].numpy(), g_len) and np.array_equal(h["out"][1].numpy(), g_tok))
        return g_len, {"outputs_valid": ok, "host_entry_point_matches": same}

    def host_buffers(self):
        if getattr(self, "_host", None) is None:
            torch, w = self.torch, self.w
            pin = lambda a, bf=False: (torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16) if bf
                                       else torch.from_numpy(np.ascontiguousarray(a))).pin_memory()
            h_draft = None if self.draft is None else pin(w.draft, self.is_bf16)
            h_lens = None if w.lens is None else pin(w.lens)
            inputs = (pin(w.target, self.is_bf16), h_draft, pin(w.tokens), h_lens,
                      None if self.greedy else pin(w.uniforms))
            out = (torch.empty(w.B, dtype=torch.int32).pin_memory(),
                   torch.empty(w.B, w.k_max + 1, dtype=torch.int32).pin_memory())
            n = self.sv.host_staging_bytes(w.B, w.k_max, w.V, self.sv.BF16 if self.is_bf16 else self.sv.F32,
                                           has_draft=h_draft is not None, has_lens=h_lens is not None)
            self._host = {"inputs": inputs, "out": out,
                          "staging": torch.empty(max(n, 256), dtype=torch.uint8, device=self.dev)}
        return self._host

    def release(self):
        for name in ("target", "draft", "tokens", "lens", "uniforms", "out", "ws", "_host"):
            setattr(self, name, None)


def reread_bytes(w, g_len, greedy=False) -> int:
    """Algorithmic bytes of the final draw: the target row j again, plus the
    draft row j when a draft with logits was rejected there (greedy: none)."""
    if greedy:
        return 0
    L = w.draft_lens
    resid = (g_len < L) & (w.draft is not None)
    return int((1 + resid.astype(np.int64)).sum()) * w.V * w.esize


def draw_path_of(sv, w, greedy, forced=0) -> str:
    """The draw path a call takes for this workload: `forced` (a DrawPath)
    or else the library's AUTO choice ("cluster" or "queue"; greedy calls
    make no draw)."""
    if greedy:
        return "none"
    if forced:
        return "cluster" if forced == sv.DrawPath.CLUSTER else "queue"
    dt = sv.BF16 if w.dtype == "bf16" else sv.F32
    path = sv.auto_draw_path(w.B, w.k_max, w.V, dt, w.target.shape[2])
    return "cluster" if path == sv.DrawPath.CLUSTER else "queue"


def launches_per_call(B: int, path: str, draft_logits: bool) -> int:
    """Kernels one spec_verify call launches: the control-word zeroing
    kernel, the row-statistics kernel per block of up to 4096 requests, then
    the scan kernel alone (greedy), the cluster kernel (scan and draw, small
    batches), or the scan kernel, the draw kernel and (with draft logits:
    residual draws) the selection kernel."""
    n = 1 + math.ceil(B / MAX_REQUESTS_PER_STATS_LAUNCH)
    if path in ("none", "cluster"):
        return n + 1
    return n + 2 + int(draft_logits)


def config_record(dw, cfg, steps, warmup, k1_samples, peak):
    """Per-workload figures for the per_config block of the bench line."""
    w = dw.w
    dev_ms = dw.time_steps(steps, warmup)
    k1 = dw.time_k1(k1_samples)
    g_len, parity = dw.host_check()
    alg = stats_pass_bytes(w, dw.greedy)
    rr = reread_bytes(w, g_len, dw.greedy)
    step_ms = dev_ms / steps
    k1_med, k1_mean = float(np.median(k1)), statistics.fmean(k1)
    return {
        "workload": workload_desc(w, cfg)["workload"], "l2": dw.l2_note, "steps": steps,
        "positions_per_s": w.positions * steps / (dev_ms / 1e3),
        "step_us": 1e3 * step_ms, "step_gbs": alg / (step_ms / 1e3) / 1e9,
        "step_frac": alg / (step_ms / 1e3) / 1e9 / peak,
        "step_gbs_with_reread": (alg + rr) / (step_ms / 1e3) / 1e9,
        "stats_bytes": alg, "reread_bytes": rr,
        "k1_samples": len(k1), "k1_us_median": 1e3 * k1_med, "k1_us_mean": 1e3 * k1_mean,
        "k1_gbs_median": alg / (k1_med / 1e3) / 1e9, "k1_frac_median": alg / (k1_med / 1e3) / 1e9 / peak,
        "k1_frac_mean": alg / (k1_mean / 1e3) / 1e9 / peak,
        "accept_rate": float(g_len.sum() / max(1, w.positions)), "mean_accept_len": float(g_len.mean()),
        "draw_path": draw_path_of(dw.sv, w, dw.greedy, dw.draw_path), "parity": parity,
    }


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
    greedy = bool(args.greedy)
    kernel = {"auto": sv.StatsKernel.AUTO, "tma": sv.StatsKernel.TMA, "vec16": sv.StatsKernel.VEC16,
              "scalar": sv.StatsKernel.SCALAR}[args.stats_kernel]
    stream = torch.cuda.current_stream()
    peak, peak_kind = measured_peak()
    w = make_rank_workload(args.config, rank)
    draw_path = {"auto": sv.DrawPath.AUTO, "queue": sv.DrawPath.QUEUE, "cluster": sv.DrawPath.CLUSTER}[args.draw_path]
    dw = DeviceWorkload(sv, torch, dev, stream, w, greedy, kernel, draw_path)

    K, W = args.steps, args.warmup
    with ClockSampler(local_rank) as clocks:
        t_rank = dw.time_steps(K, W, barrier)
    region_ms = t_rank
    t_max = max_over_ranks(t_rank, dev)
    positions = w.positions
    value = aggregate_value(n, positions, K, t_max)
    ms_per_step = t_max / K

    # the row-statistics kernel alone, in its own pass of at least 10 launches
    k1_ms = dw.time_k1(max(args.k1_samples, 10))
    g_len, parity = dw.host_check()
    assert parity["outputs_valid"], "timed run produced invalid outputs"
    assert parity["host_entry_point_matches"], "host entry point disagrees with device entry point"
    accept_rate = float(g_len.sum() / max(1, positions))

    # ---------------- end to end through the host entry point ----------------
    e2e = None
    if args.e2e_steps > 0:
        h = dw.host_buffers()

        def e2e_step():
            sv.spec_verify_host(*h["inputs"], w.temperature, greedy, V=w.V, out=h["out"], staging=h["staging"],
                                workspace=dw.ws, stream=stream)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.e2e_steps)]
        barrier()
        torch.cuda.synchronize()
        for a, b in ev:
            a.record(stream)
            e2e_step()
            b.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev)
        assert np.array_equal(h["out"][0].numpy(), g_len), "host entry point disagrees with device entry point"
        e2e = {"value": aggregate_value(n, positions, args.e2e_steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": host_copy_bytes(w, greedy),
               "d2h_bytes_per_step": int(h["out"][0].nbytes + h["out"][1].nbytes),
               "steps": args.e2e_steps, "ms_per_step": e2e_ms / args.e2e_steps}

    # ---------------- roofline of the row-statistics kernel ----------------
    alg = stats_pass_bytes(w, greedy)
    rr = reread_bytes(w, g_len, greedy)
    k1_mean, k1_med = statistics.fmean(k1_ms), float(np.median(k1_ms))
    achieved = alg / (k1_mean / 1e3) / 1e9
    variant = "tma" if args.stats_kernel == "auto" else args.stats_kernel
    traffic = committed_traffic(variant, args.config)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": traffic, "peak_kind": f"{peak_kind} (copy bandwidth, MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback 6650 GB/s",
                "kernel": f"row_stats ({variant})", "algorithmic_bytes_per_launch": alg,
                "kernel_ms": k1_mean, "kernel_ms_median": k1_med,
                "kernel_ms_p10": float(np.percentile(k1_ms, 10)), "kernel_samples": len(k1_ms),
                "frac_median": alg / (k1_med / 1e3) / 1e9 / peak,
                "whole_step_gbs": alg / (ms_per_step / 1e3) / 1e9,
                "whole_step_frac": alg / (ms_per_step / 1e3) / 1e9 / peak,
                "reread_bytes_per_step": rr,
                "whole_step_gbs_with_reread": (alg + rr) / (ms_per_step / 1e3) / 1e9,
                "whole_step_frac_with_reread": (alg + rr) / (ms_per_step / 1e3) / 1e9 / peak,
                # context: B200's nominal HBM3e bandwidth (8.0 TB/s), not the denominator
                "frac_of_nominal_8000": achieved / NOMINAL_HBM_GBS,
                "whole_step_frac_of_nominal_8000": alg / (ms_per_step / 1e3) / 1e9 / NOMINAL_HBM_GBS}

    cfgd = workload_desc(w, args.config)
    cfgd.update({"parallelism": f"replicas{n}" if n > 1 else "single",
                 "sharding": "each rank verifies its own batch; no data-path collective",
                 "l2": dw.l2_note, "stats_kernel": variant, "greedy": greedy,
                 "draw_path": draw_path_of(sv, w, greedy, draw_path)})
    dw.release()

    # ---------------- the other workloads (rank 0, N = 1) ----------------
    per_config = None
    if rank == 0 and n == 1 and not args.no_per_config:
        per_config = {}
        for cfg in sorted(CONFIGS):
            if cfg == args.config:
                continue
            wc = make_rank_workload(cfg, 0)
            dc = DeviceWorkload(sv, torch, dev, stream, wc, greedy, kernel, draw_path)
            per_config[str(cfg)] = config_record(dc, cfg, args.per_config_steps, max(W, 3),
                                                 max(args.k1_samples, 10), peak)
            dc.release()
            del dc
            torch.cuda.empty_cache()

    # ---------------- CPU oracle baseline (rank 0, N = 1) ----------------
    cpu = None
    if rank == 0 and n == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(w, args.cpu_seconds, greedy)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": n, "steps": K, "warmup": W,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic", "config": cfgd,
            "e2e": e2e, "gpu_launches": K * launches_per_call(w.B, draw_path_of(sv, w, greedy, draw_path), w.draft is not None), "roofline": roofline,
            "cpu_baseline": cpu, "clocks": clocks.summary(),
            "hbm_gbs": alg / (ms_per_step / 1e3) / 1e9,
            "accept_rate": accept_rate, "mean_accept_len": float(g_len.mean()),
            "parity": parity,
            "timing": {"region_ms": region_ms, "k1_event_samples": len(k1_ms),
                       "k1_pass": "separate pass after the timed region, events around the row-statistics "
                                  "kernel only"},
            "per_config": per_config,
        }
        print(json.dumps(line), flush=True)
    if n > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
