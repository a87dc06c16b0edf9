"""Benchmark of the KVzip compression hot path on B200.

One step = score (pass 1 row log-sum-exp + pass 2 context-key column max, in
passes of 4096 input positions) -> select (top 25% per head) -> compact (the
kept K/V rows packed in place) over a whole Qwen2.5-14B-shaped context: 48
layers x 8 KV heads, G=5 grouped queries, d=128, n_c=131072 context keys,
32-token repeat prompt, bf16, seeded synthetic inputs resident in HBM.  The
metric is context KV pairs scored and evicted per second (B*n_c per step).
Each step starts from the same uncompacted K/V: a pristine copy is restored
before every step, outside the timed region (that 52 GB copy also leaves
nothing of the inputs in L2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload NAME] [--layers L] [--decode]

With N > 1 (launched by torch.distributed.run) every rank runs its own
independent context (different seed): weak scaling, no data-path collective.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "context KV pairs scored+evicted/sec at 1 B200; score TFLOP/s % of bf16 peak"
UNIT = "context KV pairs/s"
WORKLOAD = "qwen14b_128k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
LONG_RUN_MS = 1000.0         # timed regions at least this long are rated against the sustained bf16 peak
L2_BYTES = 126 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="kvz", choices=["kvz", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="qwen14b_128k (default, the headline), llama8b_layer, tiny, llama8b_stack, stress_ragged, "
                         "llama8b_170k_chunked, llama8b_stack_heads, llama8b_stack_int8")
    ap.add_argument("--decode", action="store_true",
                    help="also time one decode step of attention (G queries per KV head) over the pruned cache "
                         "and over the full cache; adds a 'decode' object to the JSON line")
    ap.add_argument("--layers", type=int, default=0,
                    help="run only the first L layers of the workload (a smaller case for profiling; "
                         "config.workload then names the truncation)")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        d = dict(FALLBACK_PEAKS)
        d["source"] = "fallback"
        return d


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from a committed ncu
    summary, if the kernel's source has not changed since the counters were
    taken (None otherwise)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)["%s/%s" % (kernel, workload)]
        src = os.path.join(ROOT, rec["source"])
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if h != rec["source_sha256_16"]:
            return None
        return float(rec["bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
        sm_sorted, pw = sorted(sm), sorted(power)
        return {"sm_mhz": sm_sorted[len(sm_sorted) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_median": pw[len(pw) // 2] if pw else None}


def workload_numbers(w):
    """Per-step work units of a workload, summed over its contexts."""
    B, G, d = w.B, w.G, w.d
    out = {"pairs_per_step": 0, "flops_pass1": 0, "flops_pass2": 0, "kept": 0, "select_bytes": 0}
    for c, n_c in enumerate(w.n_c):
        # (context keys, input rows) of each independently scored block: the
        # whole context, or each chunk with its own n_prompt + m_t input rows
        blocks = [(n_c, w.n_in(c))] if not w.chunk else \
            [(min(w.chunk, n_c - c0), w.n_prompt + min(w.chunk, n_c - c0)) for c0 in range(0, n_c, w.chunk)]
        vis = sum(B * G * (ni * nk + ni * (ni + 1) // 2) for nk, ni in blocks)   # pass 1 pairs
        ctx = sum(B * G * ni * nk for nk, ni in blocks)                          # pass 2 pairs
        P, free = w.n_protect, n_c - w.n_protect
        if w.mode == "heads":
            kept = int(math.floor(w.ratio * B)) * n_c
        elif w.mode == "global":
            kept = B * P + int(math.floor(w.ratio * B * free))
        else:
            kept = B * (P + int(math.floor(w.ratio * free)))
        out["pairs_per_step"] += B * n_c
        out["flops_pass1"] += 2 * d * vis
        out["flops_pass2"] += 2 * d * ctx
        out["kept"] += kept
        out["select_bytes"] += (1 if w.mode == "heads" else 5) * 4 * B * n_c
    out["flops_algorithmic"] = out["flops_pass1"]
    if w.quant:   # bf16 K, V read; int8 K, V and two fp32 scales written; idx read
        out["compact_bytes"] = out["kept"] * (d * 2 * 2 + d * 2 + 8) + 4 * out["kept"]
    else:
        out["compact_bytes"] = out["kept"] * d * 2 * 2 * 2 + 4 * out["kept"]
    return out


# ---------------------------------------------------------------------------
# oracle (CPU baseline / reference arm): bounded samples of one head
# ---------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_head_sample(head_bits, w, n_c, n_in, target_s, max_s, start_frac=0.5, block=64):
    """Time the oracle, as it stands, on one head of the workload, bounded.

    The head's bf16 inputs are decoded whole; then oracle.score runs on
    consecutive blocks of `block` input positions (all G groups) from
    `start_frac` of the input until `target_s` seconds (at most `max_s`) have
    passed; selection and compaction run on the head's partial scores.  The
    head's time is the decode + the scored rows' time scaled by the head's
    visible (row, key) pairs over theirs + select + compact.
    Returns (pairs_per_second, threads, description, seconds_spent)."""
    import numpy as np
    from oracle import kvz_oracle as orc

    Qb, Kcb, Kib, Vb = head_bits
    scale = float(np.float32(1.0 / math.sqrt(w.d)))
    t0 = time.perf_counter()
    Q, Kc, Ki = orc.bf16_bits_to_f64(Qb), orc.bf16_bits_to_f64(Kcb), orc.bf16_bits_to_f64(Kib)
    t_dec = time.perf_counter() - t0
    r0 = min(n_in - 1, int(start_frac * n_in)) // block * block
    r, t_rows, vis_rows = r0, 0.0, 0
    S = np.zeros(n_c)
    while t_rows < target_s and r < n_in and t_rows < max_s:
        r1 = min(n_in, r + block)
        t1 = time.perf_counter()
        S = np.maximum(S, orc.score(Q, Kc, Ki, scale, rows=(r, r1)))
        t_rows += time.perf_counter() - t1
        vis_rows += w.G * sum(n_c + i + 1 for i in range(r, r1))
        r = r1
    t1 = time.perf_counter()
    mode = "global" if w.mode == "global" else "per_head"
    idx, counts, offsets = orc.select(S[None, :].astype(np.float32), w.ratio, mode)
    orc.compact(Kcb[None], Vb[None], idx, counts, offsets)
    t_sc = time.perf_counter() - t1
    vis_head = orc.visible_pairs(w.G, n_c, n_in)
    t_head = t_dec + t_rows * (vis_head / vis_rows) + t_sc
    desc = ("input positions [%d, %d) of one head (all %d groups): fp64 score of those rows %.1f s, scaled x%.1f "
            "to the head's %d visible (row, key) pairs; + the head's bf16 decode %.1f s and select + compact %.2f s; "
            "value = the head's %d context pairs / that extrapolated head time"
            % (r0, r, w.G, t_rows, vis_head / vis_rows, vis_head, t_dec, t_sc, n_c))
    return n_c / t_head, _blas_threads(), desc, t_dec + t_rows + t_sc


def head_bits_of(x, h):
    import numpy as np
    import torch

    def bits(t):
        return t[h].detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return bits(x["Q"]), bits(x["K_ctx"]), bits(x["K_in"]), bits(x["V"])


def run_reference(args, w, config, rank, world):
    """The oracle on the host cores, on the same workload: each step is a
    bounded sample (a block of input positions of one head; heads cycle)."""
    import torch.distributed as dist
    from query_agnostic_kv_kvz_b200 import synth
    if rank != 0:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return
    n_ctx = len(w.n_c)
    xs = [synth.layer_inputs(w, ctx=c, seed=0, device="cpu") for c in range(n_ctx)]
    steps, warm = max(1, args.steps), max(0, args.warmup)
    # a step is sized to a few seconds so that --steps 20 --warmup 5 ends in
    # minutes; steps cycle over the contexts (a ragged batch), then the heads
    rates = [[] for _ in range(n_ctx)]
    threads, desc = 1, ""
    for s in range(warm + steps):
        c, h = s % n_ctx, (s // n_ctx) % w.H
        n_c, n_in = w.n_c[c], w.n_in(c)
        target = 2.0 if n_c * n_in * w.G > 1e9 else 1.0
        frac = ((s * 0.381966) % 1.0) * 0.98            # spread the sampled row blocks over the input
        rate, threads, desc, _ = oracle_head_sample(head_bits_of(xs[c], h), w, n_c, n_in, target, 4 * target,
                                                    start_frac=frac)
        if s >= warm:
            rates[c].append(rate)
    # the whole step: every context's B heads at that context's mean sampled rate
    t_step = sum(w.B * n_c / (sum(r) / len(r)) for n_c, r in zip(w.n_c, rates) if r)
    pairs = sum(w.B * n_c for n_c, r in zip(w.n_c, rates) if r)
    value = pairs / t_step
    ms_step = t_step * 1e3 if all(rates) else None
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": "each step: one head of layer 0 (%sheads cycle, row blocks spread over the "
                                       "input); the last step: " % ("contexts, then " if n_ctx > 1 else "") + desc +
                                       "; value and ms_per_step extrapolated to the whole step (%d heads%s)"
                                       % (w.B, " x %d contexts" % n_ctx if n_ctx > 1 else "")},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
def main():
    args = parse()
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        if args.impl == "reference":                      # the host oracle: no GPU, a CPU process group
            dist.init_process_group("gloo", timeout=timedelta(seconds=600))
        else:
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=600))

    from query_agnostic_kv_kvz_b200 import synth
    w = synth.WORKLOADS[args.workload]
    n_layers_full = w.L
    if 0 < args.layers < w.L:
        import dataclasses
        w = dataclasses.replace(w, L=args.layers)
    nums = workload_numbers(w)
    config = {"workload": "%s (L=%d, H=%d, G=%d, d=%d, n_c=%s, n_prompt=%d, keep %.2f %s%s%s)" % (
        w.name, w.L, w.H, w.G, w.d, "/".join(str(n) for n in w.n_c), w.n_prompt, w.ratio, w.mode,
        ", rows in passes of %d" % w.row_chunk if w.row_chunk else "", ", in-place compaction" if w.in_place else "")
        + ("; first %d of its %d layers only" % (w.L, n_layers_full) if w.L < n_layers_full else ""),
        "B_heads": w.B, "G": w.G, "d": w.d, "n_c": list(w.n_c), "n_in": [w.n_in(c) for c in range(len(w.n_c))],
        "ratio": w.ratio, "mode": w.mode,
        "parallelism": "replicas (weak)" if world > 1 else "single GPU"}

    if args.impl == "reference":
        run_reference(args, w, config, rank, world)
        return

    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    import query_agnostic_kv_kvz_b200 as kvz
    from query_agnostic_kv_kvz_b200.dist import max_over_ranks, rank_seed
    kvz.lib()
    stream = torch.cuda.current_stream(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    scale = float(1.0 / math.sqrt(w.d))
    ctxs = [Context(w, c, rank_seed(0, rank), dev, kvz) for c in range(len(w.n_c))]
    input_bytes = sum(c.input_bytes for c in ctxs)
    # inputs larger than L2 evict themselves (and in-place workloads restore
    # 2x their K/V between steps); smaller ones get a 256 MB write flush
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if input_bytes < 4 * L2_BYTES else None
    config["l2"] = ("inputs (%.1f GB) larger than L2%s" % (input_bytes / 1e9, "; K/V restored from a pristine copy "
                    "before every step, outside the timed events" if w.in_place else "")) if flush is None else \
        "flushed before every timed step (256 MB write, outside the timed events)"
    launches_per_step = sum(c.launches for c in ctxs)

    def prepare():
        """Untimed: restore in-place workloads' K/V; flush L2 for small inputs."""
        for c in ctxs:
            c.restore()
        if flush is not None:
            flush.zero_()

    def step(ev=False):
        """One pass of the whole path over the workload; with `ev`, returns
        event marks for pass 1, pass 2, selection and compaction."""
        marks = []

        def mark(tag):
            if ev:
                e = torch.cuda.Event(enable_timing=True)
                e.record(stream)
                marks.append((tag, e))
        for c in ctxs:
            H = w.H
            for l in range(w.L):
                Kl = c.K[l * H:(l + 1) * H]
                Sl = c.S[l * H:(l + 1) * H]
                if w.chunk:
                    x = c.X[l]
                    mark("sc")
                    kvz.kvz_score_chunked(x["Q"], x["Q_tail"], Kl, x["K_in"], x["K_in_tail"], w.chunk, scale=scale,
                                          S=Sl, workspace=c.chunk_ws, status=status, stream=stream)
                    mark("end")
                    continue
                for (i0, i1) in c.chunks:
                    mark("p1")
                    kvz.kvz_score_lse2(c.Q[l], Kl, c.Kin[l], i_begin=i0, i_end=i1, scale=scale, lse2=c.lse2,
                                       ld=c.ld, workspace=c.lse_ws, status=status, stream=stream)
                    mark("p2")
                    kvz.kvz_score_colmax(c.Q[l], Kl, c.lse2, i_begin=i0, i_end=i1, scale=scale, S=Sl,
                                         accumulate=i0 > 0, status=status, stream=stream)
                    mark("end")
            mark("sel")
            if w.mode == "heads":
                kvz.kvz_head_score(c.S, S_head=c.S_head, status=status, stream=stream)
                kvz.kvz_select_heads(c.S_head, c.n_c, w.ratio, idx=c.idx, counts=c.counts, offsets=c.offsets,
                                     workspace=c.sel_ws, status=status, stream=stream)
            elif w.n_protect:
                kvz.kvz_select_protected(c.S, w.ratio, w.mode, w.n_protect, idx=c.idx, counts=c.counts,
                                         offsets=c.offsets, workspace=c.sel_ws, status=status, stream=stream)
            else:
                kvz.kvz_select(c.S, w.ratio, w.mode, idx=c.idx, counts=c.counts, offsets=c.offsets,
                               workspace=c.sel_ws, status=status, stream=stream)
            mark("cmp")
            if w.quant:
                kvz.kvz_compact_int8(c.K, c.V, c.idx, c.counts, c.offsets, Kq=c.Kq, Vq=c.Vq, K_scale=c.Ks,
                                     V_scale=c.Vs, status=status, stream=stream)
            elif w.in_place:
                kvz.kvz_compact(c.K, c.V, c.idx, c.counts, c.offsets, in_place=True, workspace=c.cmp_ws,
                                status=status, stream=stream)
            else:
                kvz.kvz_compact(c.K, c.V, c.idx, c.counts, c.offsets, K_out=c.K_out, V_out=c.V_out,
                                status=status, stream=stream)
            mark("end")
        return marks

    def phase_ms(marks):
        # "sc": one chunked-score call (both passes); booked as pass 1, pass 2 = 0
        acc = {"p1": 0.0, "p2": 0.0, "sel": 0.0, "cmp": 0.0, "sc": 0.0}
        for (tag, e0), (_, e1) in zip(marks, marks[1:]):
            if tag in acc:
                acc[tag] += e0.elapsed_time(e1)
        return [acc["p1"] + acc["sc"], acc["p2"], acc["sel"], acc["cmp"]]

    n_warm = max(3, args.warmup)
    for _ in range(n_warm):
        prepare()
        step()
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise RuntimeError("device status %d during warm-up" % int(status.item()))

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    all_marks, spans = [], []
    with ClockSampler(dev.index) as clk:
        for _ in range(args.steps):
            prepare()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            all_marks.append(step(ev=True))
            e1.record(stream)
            spans.append((e0, e1))
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    parts = [phase_ms(m) for m in all_marks]
    ms_step = sum(e0.elapsed_time(e1) for e0, e1 in spans) / len(spans)
    part_ms = [sum(p[i] for p in parts) / len(parts) for i in range(4)]
    if int(status.item()) != 0:
        raise RuntimeError("device status %d during timing" % int(status.item()))

    # ---- end to end through the host-buffer C-ABI call (kvz_compress_host):
    # every step copies the inputs in from page-locked host memory and the
    # results out, inside the timed region
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(w, ctxs, kvz, dev, stream, status, scale, ms_step)

    # ---- decode attention over the pruned cache vs the full cache (one step, all heads)
    dec = None
    if args.decode and not w.quant:
        dec = run_decode(w, ctxs[0], kvz, dev, stream, status, scale, nums)

    red = max_over_ranks([ms_step, e2e["ms"] if e2e else 0.0] + part_ms, device=dev)
    ms_step, e2e_ms, part_ms = red[0], red[1], red[2:]

    pk = peaks()
    long_run = ms_step * args.steps >= LONG_RUN_MS
    peak_tf = pk["bf16_tflops_sustained"] if long_run else pk["bf16_tflops"]
    peak_name = "%s bf16 dense, %s" % (pk["source"], "sustained (the kernel runs inside %.1f s of continuous timed work)"
                                       % (ms_step * args.steps / 1e3) if long_run else "burst")
    lse_ms, col_ms, sel_ms, cmp_ms = part_ms
    score_ms = lse_ms + col_ms
    fl1, fl2 = nums["flops_pass1"], nums["flops_pass2"]
    tf = lambda flops, ms: flops / (ms * 1e-3) / 1e12
    n_p1 = sum(w.L * (c.score_launches if w.chunk else len(c.chunks)) for c in ctxs)
    chunked = bool(w.chunk)
    achieved = tf(fl1 + fl2, lse_ms) if chunked else tf(fl1, lse_ms)
    roof = {
        "bound": "tensor",
        "kernel": ("lse_kernel + colmax_kernel (chunked score call, both passes; executed FLOP)" if chunked else
                   "lse_kernel (score pass 1: QK^T + online log-sum-exp)"),
        "achieved": achieved,
        "peak": peak_tf,
        "unit": "TFLOP/s",
        "frac": achieved / peak_tf,
        "traffic": recorded_traffic("lse_kernel", w.name) if not chunked and w.L == n_layers_full else None,
        "peak_source": peak_name,
        "frac_of_burst": achieved / pk["bf16_tflops"],
        "algorithmic_flops_per_launch": fl1 / n_p1,
        "launches_per_step": n_p1,
        "launch_ms": lse_ms / n_p1,
        "breakdown": {
            "score_pass1_ms": lse_ms, "score_pass2_ms": col_ms, "select_ms": sel_ms, "compact_ms": cmp_ms,
            "score_tflops_executed": tf(fl1 + fl2, score_ms),
            "score_frac_executed": tf(fl1 + fl2, score_ms) / peak_tf,
            "score_tflops_algorithmic": tf(nums["flops_algorithmic"], score_ms),
            "score_frac_algorithmic": tf(nums["flops_algorithmic"], score_ms) / peak_tf,
            "pass2_tflops": tf(fl2, col_ms) if col_ms > 0 else None,
            "pass2_frac": tf(fl2, col_ms) / peak_tf if col_ms > 0 else None,
            "compact_bytes": nums["compact_bytes"],
            "compact_gbs": nums["compact_bytes"] / (cmp_ms * 1e-3) / 1e9,
            "compact_frac_hbm": nums["compact_bytes"] / (cmp_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
            "select_gbs": nums["select_bytes"] / (sel_ms * 1e-3) / 1e9,
            "peaks": {"bf16_tflops_burst": pk["bf16_tflops"], "bf16_tflops_sustained": pk["bf16_tflops_sustained"],
                      "hbm_gbs": pk["hbm_gbs"], "source": pk["source"]},
        },
    }
    value = nums["pairs_per_step"] * world / (ms_step * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": n_warm, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config, "roofline": roof,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if dec is not None:
        line["decode"] = dec
    if e2e is not None:
        line["e2e"] = {"value": nums["pairs_per_step"] * world / (e2e_ms * 1e-3), "unit": UNIT,
                       "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e_ms,
                       "how": e2e["how"]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline and all(c.Q for c in ctxs):
        # one sampled head per context (a ragged batch: each context's head
        # time scaled by its B heads), the budget split over the contexts
        t_total, pairs, descs, spent, threads = 0.0, 0, [], 0.0, 1
        for ci, c in enumerate(ctxs):
            x0 = {"Q": c.Q[0], "K_ctx": c.pristine_K()[: w.H], "K_in": c.Kin[0], "V": c.pristine_V()[: w.H]}
            rate, threads, desc, sp = oracle_head_sample(head_bits_of(x0, 0), w, c.n_c, c.n_in,
                                                         12.0 / len(ctxs), 30.0 / len(ctxs))
            t_total += w.B * c.n_c / rate
            pairs += w.B * c.n_c
            spent += sp
            descs.append(("context %d (n_c=%d): " % (ci, c.n_c) if len(ctxs) > 1 else "") + "layer 0 head 0, " + desc)
        line["cpu_baseline"] = {"value": pairs / t_total, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": "; ".join(descs) + ("; value = all contexts' pairs / the sum of their "
                                                              "extrapolated times" if len(ctxs) > 1 else "") +
                                " (%.1f s of CPU time)" % spent}
        # exact ties among the GPU's scores of head 0: at the keep threshold
        # (where the lower-index rule decides) and overall (equal fp32 values)
        import numpy as np
        s0 = c.S[0].cpu().numpy()
        o0, o1 = int(c.offsets[0].item()), int(c.offsets[1].item())
        k0 = o1 - o0
        thr = np.sort(s0)[::-1][k0 - 1] if k0 > 0 else np.float32(np.inf)
        line["ties"] = {"head": 0, "at_threshold": int(np.count_nonzero(s0 == thr)) if k0 > 0 else 0,
                        "duplicate_values": int(s0.size - np.unique(s0).size)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(w, ctxs, kvz, dev, stream, status, scale, ms_step):
    """The metric through kvz_compress_host: host buffers in, host buffers
    out, the copies inside the timed region.  Per-head workloads call it once
    per layer (the heads of a layer are one context's independent problems);
    global ones once for the whole context.  Host inputs live in page-locked
    memory; when the host cannot hold every layer, the distinct layers it can
    hold are cycled (stated in `how`)."""
    import torch
    if w.chunk or w.quant or w.n_protect or w.mode == "heads" or len(ctxs) != 1:
        return None
    c = ctxs[0]
    per_layer = w.mode == "per_head"
    calls = w.L if per_layer else 1
    Bc = w.H if per_layer else w.B
    row = w.d * 2
    in_bytes = Bc * (w.G * c.n_in + 2 * c.n_c + c.n_in) * row          # Q, K_ctx, V, K_in of one call
    mode = kvz.PER_HEAD if per_layer else kvz.GLOBAL
    k = kvz.kvz_keep_count(c.n_c if per_layer else Bc * c.n_c, w.ratio)
    kept = Bc * k if per_layer else k
    out_bytes = kept * (4 + 2 * row) + Bc * 4 + (Bc + 1) * 8
    # host memory for the page-locked inputs: 60% of what is available,
    # shared by the ranks of this node
    local_ranks = max(1, int(os.environ.get("LOCAL_WORLD_SIZE", os.environ.get("WORLD_SIZE", "1"))))
    try:
        import psutil
        budget = int(0.60 * psutil.virtual_memory().available) // local_ranks
    except Exception:
        budget = (8 << 30) // local_ranks
    n_host = max(1, min(calls, (budget - 2 * out_bytes) // in_bytes))
    if n_host < calls and not per_layer:
        return None
    cudart = torch.cuda.cudart()
    registered = []

    def pinned(shape, dtype):
        # page-locked in place (torch's pinned allocator would round each
        # buffer up to a power of two); a pinned copy if registration fails
        t = torch.empty(shape, dtype=dtype)
        if t.numel() > 0:
            if int(cudart.cudaHostRegister(t.data_ptr(), t.numel() * t.element_size(), 0)) != 0:
                return t.pin_memory()
            registered.append(t)
        return t

    try:
        hosts = []
        for hl in range(n_host):
            if per_layer:
                src = {"Q": c.Q[hl], "K_ctx": c.pristine_K()[hl * w.H:(hl + 1) * w.H], "K_in": c.Kin[hl],
                       "V": c.pristine_V()[hl * w.H:(hl + 1) * w.H]}
            else:
                src = {"Q": torch.cat(c.Q), "K_ctx": c.pristine_K(), "K_in": torch.cat(c.Kin), "V": c.pristine_V()}
            h = {n: pinned(tuple(t.shape), torch.bfloat16) for n, t in src.items()}
            for n, t in src.items():
                h[n].copy_(t)
            hosts.append(h)
        outs = [{"idx": pinned((max(kept, 1),), torch.int32), "counts": pinned((Bc,), torch.int32),
                 "offsets": pinned((Bc + 1,), torch.int64), "K_out": pinned((max(kept, 1), w.d), torch.bfloat16),
                 "V_out": pinned((max(kept, 1), w.d), torch.bfloat16)} for _ in range(2)]
        ws = torch.empty(kvz.kvz_compress_host_workspace_size(Bc, w.G, c.n_c, c.n_in, w.d, w.ratio, mode),
                         dtype=torch.uint8, device=dev)
        copy_stream = torch.cuda.Stream(dev)

        def call(i):
            hx = hosts[i % n_host]
            kvz.kvz_compress_host(hx["Q"], hx["K_ctx"], hx["K_in"], hx["V"], w.ratio, mode, scale=scale,
                                  out=outs[i % 2], workspace=ws, status=status, stream=stream,
                                  copy_stream=copy_stream)

        call(0)                                             # warm-up: one call
        torch.cuda.synchronize(dev)
        steps = max(1, min(20, int(math.ceil(20000.0 / max(ms_step, 1e-3)))))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            for i in range(calls):
                call(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if int(status.item()) != 0:
            raise RuntimeError("device status %d during e2e" % int(status.item()))
        ms = e0.elapsed_time(e1) / steps
        h2d = calls * in_bytes
        d2h = calls * out_bytes
        held = ("%d distinct host layer(s)%s" % (n_host, "" if n_host == calls else
                                                  " cycled (host memory holds %d of %d)" % (n_host, calls))
                if per_layer else "the whole context's inputs in host memory")
        how = ("kvz_compress_host %s (%d heads per call, %d call(s) per step, %d timed step(s)): inputs copied in "
               "from page-locked host memory by head chunks overlapping the scoring, selection and out-of-place "
               "compaction on the device, kept rows / indices copied back; %s"
               % ("per layer" if per_layer else "for the whole context", Bc, calls, steps, held))
        return {"ms": ms, "h2d": h2d, "d2h": d2h, "how": how}
    finally:
        torch.cuda.synchronize(dev)
        for t in registered:
            cudart.cudaHostUnregister(t.data_ptr())


def run_decode(w, c, kvz, dev, stream, status, scale, nums):
    import torch
    B = w.B
    gq = torch.Generator(device=dev).manual_seed(11)
    q = torch.randn((B, w.G, w.d), generator=gq, device=dev).to(torch.bfloat16)
    if w.in_place:
        Kd, Vd = c.K.view(B * c.n_c, w.d), c.V.view(B * c.n_c, w.d)
        off_d = torch.arange(B + 1, dtype=torch.int64, device=dev) * c.n_c
    else:
        Kd, Vd, off_d = c.K_out, c.V_out, c.offsets
    full_cnt = torch.full((B,), c.n_c, dtype=torch.int32, device=dev)
    full_off = torch.arange(B + 1, dtype=torch.int64, device=dev) * c.n_c
    Kf, Vf = c.pristine_K().view(B * c.n_c, w.d), c.pristine_V().view(B * c.n_c, w.d)
    ws_d = torch.empty(kvz.lib().kvz_decode_workspace_size(B, w.G, c.n_c, w.d), dtype=torch.uint8, device=dev)
    out_d = torch.empty((B, w.G, w.d), dtype=torch.float32, device=dev)
    lse_d = torch.empty((B, w.G), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def time_decode(K_, V_, cnt, off, nbytes, iters=20):
        # a cache over twice the L2 evicts itself between steps (inputs larger
        # than L2); smaller ones get the write flush, then a read of the same
        # buffer, so that the flush's dirty lines are written back before the
        # timed call instead of inside it.  One decode call is captured in a
        # CUDA graph and replayed, so that the host-side cost of a call
        # (binding, tensor maps, two launches) does not leave the GPU idle
        # inside a short window.
        big = nbytes > 2 * L2_BYTES
        for _ in range(3):
            kvz.kvz_decode(q, K_, V_, cnt, off, c.n_c, scale=scale, out=out_d, lse2=lse_d, workspace=ws_d,
                           status=status, stream=stream)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            kvz.kvz_decode(q, K_, V_, cnt, off, c.n_c, scale=scale, out=out_d, lse2=lse_d, workspace=ws_d,
                           status=status)
        evs = []
        for _ in range(iters):            # all enqueued before one sync
            if not big:
                flush.zero_()
                flush.view(torch.float32).sum()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            evs.append((e0, e1))
        torch.cuda.synchronize(dev)
        del graph
        ts = sorted(e0.elapsed_time(e1) for e0, e1 in evs)
        return ts[len(ts) // 2]

    kept_rows = nums["kept"]
    byt = kept_rows * w.d * 2 * 2
    byt_full = B * c.n_c * w.d * 4
    t_pruned = time_decode(Kd, Vd, c.counts, off_d, byt)
    t_full = time_decode(Kf, Vf, full_cnt, full_off, byt_full)
    if int(status.item()) != 0:
        raise RuntimeError("device status %d during decode" % int(status.item()))
    pk0 = peaks()
    return {"ms": t_pruned, "bytes": byt, "gbs": byt / (t_pruned * 1e-3) / 1e9,
            "frac_hbm": byt / (t_pruned * 1e-3) / 1e9 / pk0["hbm_gbs"],
            "full_cache_ms": t_full, "full_cache_gbs": byt_full / (t_full * 1e-3) / 1e9,
            "speedup_vs_full_cache": t_full / t_pruned,
            "what": "one decode step: %d KV heads x %d grouped queries over the pruned cache (%d kept rows) vs "
                    "the full cache; median of 20 replays of a CUDA graph of the call; caches over 2x L2 "
                    "unflushed (larger than L2), smaller ones after a 256 MB write flush and a read of that "
                    "buffer" % (B, w.G, kept_rows)}


def lse_launches(B, G, n_c, i_begin, rows, sms):
    """Kernels one pass-1 call launches: lse_kernel, plus lse_merge_kernel
    when the grid's partial last wave is split (launch_lse's rule)."""
    units = B * G * ((rows + 255) // 256)
    r = units % sms
    if r == 0:
        return 1
    s = min(sms // r, ((n_c + 127) // 128 + i_begin // 128 + 1) // 8)
    if s * r > 256:
        s = 256 // r
    return 2 if s >= 2 else 1


class Context:
    """Device-resident inputs and outputs of one context of a workload: all
    layers' Q / K_in, the whole K/V cache (and, when it is compacted in
    place, a pristine copy restored before every step), scores, selection
    and outputs."""

    def __init__(self, w, c, seed, dev, kvz):
        import torch
        from query_agnostic_kv_kvz_b200 import synth
        H, G, d, L = w.H, w.G, w.d, w.L
        B = L * H
        self.w = w
        self.n_c, self.n_in = w.n_c[c], w.n_in(c)
        self.K = torch.empty((B, self.n_c, d), dtype=torch.bfloat16, device=dev)
        self.V = torch.empty((B, self.n_c, d), dtype=torch.bfloat16, device=dev)
        self.Q, self.Kin, self.X = [], [], []
        if w.chunk:
            # chunked scoring: every layer's per-chunk queries and input keys
            for l in range(L):
                x = synth.chunked_inputs(w, layer=l, ctx=c, seed=seed, device=dev)
                self.K[l * H:(l + 1) * H].copy_(x.pop("K_ctx"))
                self.V[l * H:(l + 1) * H].copy_(x.pop("V"))
                self.X.append(x)
            self.chunk_ws = torch.empty(kvz.kvz_score_chunked_workspace_size(H, G, self.n_c, w.n_prompt, w.chunk),
                                        dtype=torch.uint8, device=dev)
            n_full, tail = self.n_c // w.chunk, self.n_c % w.chunk
            self.score_launches = (1 if n_full else 0) + (1 if tail else 0)     # lse launches per layer
        for l in range(L if not w.chunk else 0):
            x = synth.layer_inputs(w, layer=l, ctx=c, seed=seed, device=dev)
            self.K[l * H:(l + 1) * H].copy_(x["K_ctx"])
            self.V[l * H:(l + 1) * H].copy_(x["V"])
            self.Q.append(x["Q"])
            self.Kin.append(x["K_in"])
            del x
        self.K0 = self.K.clone() if w.in_place else None
        self.V0 = self.V.clone() if w.in_place else None
        self.input_bytes = 2 * self.K.numel() * 2 + sum(t.numel() * 2 for t in self.Q + self.Kin)
        chunk = min(w.row_chunk or self.n_in, self.n_in)
        self.chunks = [(i0, min(self.n_in, i0 + chunk)) for i0 in range(0, self.n_in, chunk)]
        self.ld = (chunk + 255) // 256 * 256
        self.lse2 = torch.empty((H, G, self.ld), dtype=torch.float32, device=dev)
        self.lse_ws = torch.empty(kvz.kvz_score_lse2_workspace_size(), dtype=torch.uint8, device=dev)
        self.S = torch.empty((B, self.n_c), dtype=torch.float32, device=dev)
        mode = kvz.GLOBAL if w.mode == "global" else kvz.PER_HEAD
        if w.mode == "heads":
            cap = max(1, kvz.kvz_keep_count(B, w.ratio) * self.n_c)
            self.S_head = torch.empty(B, dtype=torch.float32, device=dev)
            self.sel_ws = torch.empty(kvz.lib().kvz_select_heads_workspace_size(B), dtype=torch.uint8, device=dev)
        else:
            free = self.n_c - w.n_protect
            if mode == kvz.GLOBAL:
                cap = max(1, B * w.n_protect + kvz.kvz_keep_count(B * free, w.ratio))
            else:
                cap = max(1, B * (w.n_protect + kvz.kvz_keep_count(free, w.ratio)))
            self.sel_ws = torch.empty(kvz.kvz_select_workspace_size(B, self.n_c, mode), dtype=torch.uint8,
                                      device=dev)
        self.idx = torch.empty(cap, dtype=torch.int32, device=dev)
        self.counts = torch.empty(B, dtype=torch.int32, device=dev)
        self.offsets = torch.empty(B + 1, dtype=torch.int64, device=dev)
        self.cmp_ws = torch.empty(kvz.kvz_compact_workspace_size(B, self.n_c), dtype=torch.uint8, device=dev)
        if w.quant:
            self.Kq = torch.empty((cap, d), dtype=torch.int8, device=dev)
            self.Vq = torch.empty((cap, d), dtype=torch.int8, device=dev)
            self.Ks = torch.empty(cap, dtype=torch.float32, device=dev)
            self.Vs = torch.empty(cap, dtype=torch.float32, device=dev)
        elif not w.in_place:
            self.K_out = torch.empty((cap, d), dtype=torch.bfloat16, device=dev)
            self.V_out = torch.empty((cap, d), dtype=torch.bfloat16, device=dev)
        # lse (+ colmax, + S fill on the first chunk) per (layer, chunk); select 10 (1 per head
        # when one CTA per head does it); compact 1 (in place: workspace fill, reader-run
        # pre-pass, compaction)
        per_head_one = w.mode == "per_head" and (self.n_c <= 49152 or B >= 128)
        # head level: fill + head max, one-segment selection (1 launch up to 49152 heads), csr + idx
        sel = 1 if per_head_one else (5 if w.mode == "heads" else 10)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        if w.chunk:   # per layer: fill, then for the full chunks and the tail: pass 1 (+ merge) and pass 2
            T, tail = self.n_c // w.chunk, self.n_c % w.chunk
            per_layer = 1 + (lse_launches(H * T, G, w.chunk, 0, w.n_prompt + w.chunk, sms) + 1 if T else 0) + \
                (lse_launches(H, G, tail, 0, w.n_prompt + tail, sms) + 1 if tail else 0)
        else:         # per layer: fill, then per row pass: pass 1 (+ merge) and pass 2
            per_layer = 1 + sum(lse_launches(H, G, self.n_c, i0, i1 - i0, sms) + 1 for i0, i1 in self.chunks)
        self.launches = L * per_layer + sel + (3 if w.in_place else 1)

    def restore(self):
        if self.K0 is not None:
            self.K.copy_(self.K0)
            self.V.copy_(self.V0)

    def pristine_K(self):
        return self.K0 if self.K0 is not None else self.K

    def pristine_V(self):
        return self.V0 if self.V0 is not None else self.V


if __name__ == "__main__":
    main()
