#!/usr/bin/env python
"""Throughput of the flow-map block draft + prefix verify step on B200.

One step = one speculative round of the hot path for every sequence of the
workload: append the round's new target-feature rows to the context cache
(fm_project_context), draft one K=16 block per noise sample (fm_draft) and
verify it against target logits (fm_verify_greedy / fm_verify_sample).
Inputs are seeded synthetic arrays (fm_synth) with the workload's shapes;
the target model itself is not run: synthetic target logits stand in for
its scores.

Prints one JSON line (rank 0).  `value` is drafted 16-token blocks per
second over all ranks (each rank runs its own replica: weak scaling, no
collective on the data path); `verified_tokens_per_s` counts accepted
tokens plus the target's correction/bonus token.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle on host cores
"""
from __future__ import annotations

import argparse
import faulthandler
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import fm_synth as fs  # noqa: E402

METRIC = "drafted 16-token blocks/s + verified tokens/s on 1 B200; % of HBM/TC roofline"
DEFAULT_WORKLOAD = "qwen3_8b_bs1"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="fm", choices=["fm", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(fs.WORKLOADS))
    ap.add_argument("--rounds", type=int, default=0, help="distinct seeded rounds cycled (0: auto)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of CUDA graphs")
    ap.add_argument("--profile-all", action="store_true", help="log per-class kernel times")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--factorised", action="store_true",
                    help="also draft every round factorised (position i from its own noise "
                         "block) and report both accepted-length histograms (untimed)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ---------------------------------------------------------------- clocks
def _clock_child(bus: str, conn, stop) -> None:
    """Sampler process: SM clock and throttle reasons through NVML as fast as
    the calls return (a separate process, so the timing loop's GIL does not
    starve it); sends [(t_before, t_after, mhz, reasons)] on stop."""
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        conn.send(("ready", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)))
    except Exception as e:  # pragma: no cover
        conn.send(("error", str(e)))
        return
    out = []
    while not stop.is_set():
        t0 = time.monotonic()
        try:
            mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception:
            continue
        out.append((t0, time.monotonic(), mhz, r))
        time.sleep(0.0002)
    conn.send(out)


def window_samples(raw, t0: float, t1: float, reasons: dict):
    """SM clocks and throttle-reason names of the NVML samples taken in the
    timed region [t0, t1].  A sample is the interval [before, after] of its
    two NVML calls; one that overlaps the region counts (an NVML call can
    take longer than a short timed region, which then holds no sample that
    started and ended inside it)."""
    mhz_in, names = [], set()
    for tb, ta, mhz, r in raw:
        if ta >= t0 and tb <= t1:
            mhz_in.append(mhz)
            for bit, name in reasons.items():
                if r & bit:
                    names.add(name)
    return mhz_in, names


class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region by a
    separate NVML process; the samples overlapping [enter, exit] count."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_dev: int):
        self.samples, self.reasons, self.ok, self.window = [], set(), False, 0.0
        self.err = ""
        try:
            import multiprocessing as mp
            import torch
            pr = torch.cuda.get_device_properties(torch_dev)
            bus = "%08X:%02X:%02X.0" % (int(pr.pci_domain_id), int(pr.pci_bus_id),
                                        int(pr.pci_device_id))
            mctx = mp.get_context("spawn")
            self.stop = mctx.Event()
            self.conn, child = mctx.Pipe()
            self.proc = mctx.Process(target=_clock_child, args=(bus, child, self.stop), daemon=True)
            self.proc.start()
            if not self.conn.poll(60):
                raise RuntimeError("clock sampler did not start")
            tag, val = self.conn.recv()
            if tag != "ready":
                raise RuntimeError(val)
            self.max_mhz = val
            self.ok = True
        except Exception as e:  # pragma: no cover
            self.err = str(e)

    def __enter__(self):
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *a):
        self.t1 = time.monotonic()
        if not self.ok:
            return
        self.stop.set()
        raw = self.conn.recv() if self.conn.poll(30) else []
        self.proc.join(10)
        self.window = self.t1 - self.t0
        self.samples, self.reasons = window_samples(raw, self.t0, self.t1, self.REASONS)


    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable: " + self.err]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "window_ms": round(1e3 * self.window, 1)}


# ---------------------------------------------------------------- algorithmic bytes
def _strip_comments(text: str) -> str:
    """C/C++/CUDA source without comments and blank lines (string and
    character literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).splitlines())
    return "\n".join(ln for ln in lines if ln)


def source_sha1(root: str = ROOT) -> str:
    """Hash of the kernel sources without comments; a stored ncu traffic
    figure is reported only while it matches (the kernels have not changed
    since the capture)."""
    import hashlib
    h = hashlib.sha1()
    csrc = os.path.join(root, "step_flow_map_b200", "csrc")
    for f in sorted(os.listdir(csrc)) + ["../../include/flashmap.h"]:
        with open(os.path.join(csrc, f), encoding="utf-8") as fh:
            h.update(f.encode() + _strip_comments(fh.read()).encode())
    return h.hexdigest()


def stored_traffic(kernel: str, workload: str, path: str | None = None):
    """DRAM bytes per launch from profiles/traffic.txt (JSON), or None."""
    p = path or os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(workload)
    if e and e.get("source_sha1") == source_sha1():
        return e["dram_bytes_per_launch"]
    return None


RANK_SEED_STRIDE = 100000   # round seeds of rank k start at k * stride: replicas see distinct inputs


def round_seed(i: int, rank: int) -> int:
    """Seed index of the i-th distinct round of a rank."""
    return i + RANK_SEED_STRIDE * rank


def reduce_over_ranks(dist, device, ms: float, verified: float, world: int):
    """Whole-job figures of the replicas: the slowest rank's device time and
    the sum of verified tokens (each rank drafts its own sequences; no
    exchange on the data path).  `dist` None means one process."""
    if dist is None:
        return ms, verified * world
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    v = torch.tensor([float(verified)], dtype=torch.float64, device=device)
    dist.all_reduce(v)
    return float(t.item()), float(v.item())


def acceptance_stats(n, K: int) -> dict:
    """Accepted-length statistics of timed rounds: `n` holds one accepted
    length (0..K) per (round, sequence).  hist[i] = rounds with n = i;
    p_reach[i-1] = P(n >= i), the chance the verifier reaches draft position
    i with every earlier position accepted."""
    a = np.asarray(n, dtype=np.int64).reshape(-1)
    hist = np.bincount(np.clip(a, 0, K), minlength=K + 1)
    tot = max(int(a.size), 1)
    reach = [round(float((a >= i).sum()) / tot, 4) for i in range(1, K + 1)]
    return {"mean": round(float(a.mean()) if a.size else 0.0, 3),
            "hist": [int(x) for x in hist], "p_reach": reach}


def workload_config(w: fs.Workload, rounds: int, world: int) -> dict:
    """The `config` object of both arms' JSON lines."""
    s = w.shape
    step_bytes = sum(v for k, v in algorithmic_bytes(w).items() if not k.endswith("_per_launch"))
    return {"workload": w.name, "sequences_per_gpu": w.B, "noise_drafts": w.n_noise, "K": s.K,
            "V": s.V, "d": s.d, "n_blocks": s.n_blocks, "context_rows": w.ctx + w.new_rows,
            "num_steps": len(w.t_grid) - 1, "temperatures": sorted(set(w.temps)),
            "distinct_rounds": rounds, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2: every step streams ~%.2f GB" % (step_bytes / 1e9)}


def algorithmic_flops(w: fs.Workload):
    """FLOPs of each kernel class per step (2 per multiply-add)."""
    s = w.shape
    M, V, d, F, nb = w.M, s.V, s.d, s.mlp, s.n_blocks
    steps = len(w.t_grid) - 1
    ctx_rows = w.ctx + w.new_rows
    dit_params = nb * (3 * d * d + d * d + 2 * d * F)
    attn = nb * 4 * M * (ctx_rows + s.K) * d          # QK^T and PV over context + block
    return {"embed": 2 * M * V * d * steps, "lm_head": 2 * M * V * d * steps,
            "dit_gemm": 2 * M * dit_params * steps, "attn": attn * steps}


def persistent_pass(w: fs.Workload) -> bool:
    """True when the library runs the DiT as its persistent pass (one
    sequence, one noise draft, bf16, 128-wide heads) and so projects the
    round's new context rows inside that pass's QKV phases, with the key and
    value weights it streams anyway."""
    s = w.shape
    return (w.dtype == "bf16" and w.B == 1 and w.n_noise == 1 and s.K == 16 and s.dh == 128
            and s.K + w.new_rows <= 64)


def algorithmic_bytes(w: fs.Workload):
    """Bytes each kernel class must move per step (weights, activations, caches)."""
    s = w.shape
    e = 2 if w.dtype == "bf16" else 4
    M = w.M
    V, d, F, nb = s.V, s.d, s.mlp, s.n_blocks
    steps = len(w.t_grid) - 1
    ctx_rows = w.ctx + w.new_rows
    n_part = (V + 127) // 128
    embed = V * d * e + M * V * e + 2 * M * d * 4                     # E, noise/D, x and z
    lm = V * d * e + M * d * e + M * n_part * 8                        # W_lm, h, argmax partials
    if any(t > 0 for t in w.temps) or steps > 1:
        lm = V * d * e + M * d * e + M * V * 4                         # logits written
    dit = nb * (3 * d * d + d * d + 2 * d * F) * e                     # block weights
    attn = nb * w.B * ctx_rows * 2 * d * e                             # context keys/values
    ctx = (w.B * w.new_rows * (s.n_taps * s.hidden * e + d * 4)
           + s.n_taps * s.hidden * d * e)                              # hidden rows, fc
    if w.new_rows and not persistent_pass(w):
        ctx += nb * 2 * d * d * e    # K/V weights of a separate projection; inside the persistent
        #                              pass they are the QKV weights the DiT already streams
    verify = w.B * w.n_noise * (s.K + 1) * V * 4
    return {"embed": embed * steps, "lm_head": lm * steps, "dit_gemm": dit * steps,
            "attn": attn * steps, "context": ctx, "verify": verify,
            "embed_per_launch": embed, "lm_head_per_launch": lm}


# ---------------------------------------------------------------- GPU arm
def run_fm(args, w, rank, world, local_rank):
    import torch
    import step_flow_map_b200 as fmb
    from step_flow_map_b200.host import Context, to_device

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    s = w.shape
    B, N, K, V = w.B, w.n_noise, s.K, s.V
    seqs = list(range(B))
    sampled = [b for b in seqs if w.temps[b] > 0]
    greedy = [b for b in seqs if w.temps[b] == 0]
    # contiguous halves only (greedy first, then sampled), as in the mixed workload
    assert sampled == list(range(len(greedy), B)) or not sampled
    t_setup = time.time()
    log(f"{w.name}: generating weights")
    W = fs.make_weights(s, w.dtype)
    log("loading context")
    max_new = max(1, min(1024, w.ctx))
    factorised = args.factorised and B <= 4 and all(t == 0 for t in w.temps)
    ctx = Context(s, w.dtype, W, max_ctx=w.ctx + max(w.new_rows, 1) + 8, max_seqs=B,
                  max_noise=max(N, s.K) if factorised else N, max_new=max(max_new, w.new_rows))
    del W
    for b in seqs:
        h = fs.prefill_hidden(w, b)
        for p0 in range(0, w.ctx, max_new):
            ctx.project([b], to_device(h[p0:p0 + max_new][None], w.dtype), [p0])
    torch.cuda.synchronize()
    log("prefill done")
    stream = torch.cuda.current_stream()

    per_round_mb = (B * N * K * V * (2 if w.dtype == "bf16" else 4) + B * N * (K + 1) * V * 4) / 2**20
    R = args.rounds or min(w.rounds, args.steps + args.warmup, 32, max(1, int(4096 // per_round_mb)))
    R = max(1, R)
    need_logits = bool(sampled)
    tokens = torch.empty((B, N, K), dtype=torch.int32, device="cuda")
    dlog = torch.empty((B, N, K, V), dtype=torch.float32, device="cuda") if need_logits else None
    rounds = []
    for i in range(R):
        r = round_seed(i, rank)
        ri = fs.round_inputs(w, r)
        rd = {"noise": to_device(ri.noise, w.dtype),
              "hidden": to_device(ri.new_hidden, w.dtype) if w.new_rows else None,
              "u_draft": to_device(ri.u_draft), "u_accept": to_device(ri.u_accept),
              "u_res": to_device(ri.u_res)}
        # untimed pass: the drafted block the synthetic target scores
        if w.new_rows:
            ctx.project(seqs, rd["hidden"], [w.ctx] * B)
        lg = torch.empty((B, N, K, V), dtype=torch.float32, device="cuda")
        fmb.fm_draft(ctx.ctx, seqs, rd["noise"], N, w.t_grid, w.temps, rd["u_draft"], tokens, lg,
                     stream)
        tgt = fs.target_logits(w, r, tokens.cpu().numpy(), lg.cpu().numpy())
        del lg
        rd["target"] = to_device(tgt)
        rounds.append(rd)
    n_acc_round = torch.zeros((R, B), dtype=torch.int32, device="cuda")
    branch = torch.empty(B, dtype=torch.int32, device="cuda")
    out_tok = torch.empty((B, K + 1), dtype=torch.int32, device="cuda")
    g, h0 = len(greedy), len(greedy)

    def step(rd, n_acc, st, outs=None):
        br, ot = outs if outs is not None else (branch, out_tok)
        if w.new_rows:
            fmb.fm_project_context(ctx.ctx, seqs, rd["hidden"], w.new_rows, [w.ctx] * B, st)
        fmb.fm_draft(ctx.ctx, seqs, rd["noise"], N, w.t_grid, w.temps, rd["u_draft"], tokens, dlog,
                     st)
        tgt = rd["target"]
        if g:
            fmb.fm_verify_greedy(ctx.ctx, tgt, tokens, g, N, K, V, n_acc, br, ot, st)
        if sampled:
            ns = B - g
            fmb.fm_verify_sample(ctx.ctx, tgt[h0:], dlog[h0:], tokens[h0:], ns, N, K, V,
                                 w.temps[h0], rd["u_accept"][h0:], rd["u_res"][h0:],
                                 n_acc[h0:], br[h0:], ot[h0:], st)

    def barrier():
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        if dist is None:
            return x
        t = torch.tensor([x], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    setup_s = time.time() - t_setup
    log(f"{R} rounds prepared in {setup_s:.1f} s; timing")
    for k in range(args.warmup):
        step(rounds[k % R], n_acc_round[k % R], stream)
    # untimed eager pass with every kernel class between CUDA events (the
    # event pairs serialise neighbours): the per-class shares, and which
    # class dominates the step
    n_eager = 20 if args.profile_all else 3
    fmb.fm_profile(ctx.ctx, (1 << fmb.FM_PROF_N) - 1)
    fmb.fm_profile_read(ctx.ctx, reset=True)
    for k in range(n_eager):
        step(rounds[k % R], n_acc_round[k % R], stream)
    torch.cuda.synchronize()
    pm, pl = fmb.fm_profile_read(ctx.ctx, reset=True)
    fmb.fm_profile(ctx.ctx, 0)
    eager = {name: {"us_per_step": round(pm[i] / n_eager * 1e3, 1),
                    "launches_per_step": round(pl[i] / n_eager, 2)}
             for name, i in fmb.FM_PROF.items() if pl[i]}
    for name, e in eager.items():
        log(f"eager profile {name:9s}: {e['us_per_step']:8.1f} us/step, "
            f"{e['launches_per_step']:.0f} launches/step")
    ab = algorithmic_bytes(w)
    candidates = ["embed", "lm_head", "dit_gemm", "attn"]
    dominant = max((c for c in candidates if c in eager), key=lambda c: eager[c]["us_per_step"])
    # only the dominant class carries event pairs, inside the timed graphs
    # when it has few launches per step; a class of many short launches
    # (event pairs break their programmatic overlap) is timed in separate
    # replays of the same step instead
    prof_classes = [dominant]
    mask = 1 << fmb.FM_PROF[dominant]
    inline_events = eager[dominant]["launches_per_step"] <= 8
    barrier()
    # one CUDA graph per distinct round
    fmb.fm_profile(ctx.ctx, mask if inline_events else 0)
    fmb.fm_profile_read(ctx.ctx, reset=True)
    graphs = []
    if not args.no_graph:
        for i in range(R):
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                step(rounds[i], n_acc_round[i], torch.cuda.current_stream())
            graphs.append(gr)
        _, cap_launches = fmb.fm_profile_read(ctx.ctx, times=False)
        launches_per_step = sum(cap_launches) / R
        for gr in graphs:          # one untimed replay each
            gr.replay()
        barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        ev0.record(stream)
        for k in range(args.steps):
            i = (args.warmup + k) % R
            if graphs:
                graphs[i].replay()
            else:
                step(rounds[i], n_acc_round[i], stream)
        ev1.record(stream)
        torch.cuda.synchronize()
    prof_ms, launches = fmb.fm_profile_read(ctx.ctx, reset=True)
    fmb.fm_profile(ctx.ctx, 0)
    if not graphs:
        launches_per_step = sum(launches) / args.steps
        timed_steps = args.steps
    else:
        timed_steps = R   # each graph's event pairs hold its last replay
    if not inline_events:
        fmb.fm_profile(ctx.ctx, mask)
        fmb.fm_profile_read(ctx.ctx, reset=True)
        if graphs:
            pgraphs = []
            for i in range(R):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr):
                    step(rounds[i], n_acc_round[i], torch.cuda.current_stream())
                pgraphs.append(gr)
            _, cap_launches = fmb.fm_profile_read(ctx.ctx, times=False)
            for gr in pgraphs:
                gr.replay()
        else:
            for k in range(R):
                step(rounds[k], n_acc_round[k], stream)
        torch.cuda.synchronize()
        prof_ms, launches = fmb.fm_profile_read(ctx.ctx, reset=True)
        fmb.fm_profile(ctx.ctx, 0)
        timed_steps = R
        if graphs:
            del pgraphs
    barrier()
    n_all = n_acc_round.cpu().numpy()          # [R, B] accepted lengths
    n_round = n_all.sum(axis=1)
    n_sum = int(sum(n_round[(args.warmup + k) % R] for k in range(args.steps)))
    acc = acceptance_stats(np.stack([n_all[(args.warmup + k) % R] for k in range(args.steps)]), K)
    verified = n_sum + args.steps * B           # accepted + one target token per sequence
    ms, verified = reduce_over_ranks(dist, "cuda", ev0.elapsed_time(ev1), verified, world)
    sec = ms / 1e3
    blocks = B * N * args.steps * world
    value = blocks / sec
    tok_per_s = verified / sec

    # roofline of the dominant kernel class (largest timed share).  The DiT
    # class is one persistent launch per step (block weights and the
    # context keys/values with the attention inside it) or one launch per
    # GEMM, reported as their mean.
    pk, pk_kind = peaks()
    af = algorithmic_flops(w)
    n_steps = len(w.t_grid) - 1
    ridge = pk["bf16_tflops_sustained"] * 1e12 / (pk["hbm_gbs"] * 1e9)
    per_class = {}
    for c in prof_classes:
        i = fmb.FM_PROF[c]
        if prof_ms[i] <= 0 or launches[i] == 0:
            continue
        per_step = launches[i] / timed_steps
        if graphs:
            per_step = cap_launches[i] / R
        avg = prof_ms[i] / timed_steps / per_step
        step_b, step_f = ab[c], af.get(c, 0)
        kern = c
        if c == "dit_gemm" and round(per_step) == n_steps:
            kern = "k_dit_persistent"
            step_b += ab["attn"]
            step_f += af["attn"]
        b_l, f_l = step_b / per_step, step_f / per_step
        tensor = f_l / max(b_l, 1) > ridge
        ach = (f_l / (avg / 1e3) / 1e12) if tensor else (b_l / (avg / 1e3) / 1e9)
        peak = pk["bf16_tflops_sustained"] if tensor else pk["hbm_gbs"]
        per_class[c] = {"kernel": kern, "launches_per_step": round(per_step, 2),
                        "ms_per_launch": round(avg, 5), "bytes_per_launch": int(b_l),
                        "flops_per_launch": int(f_l), "bound": "tensor" if tensor else "hbm",
                        "achieved": round(ach, 1), "unit": "TFLOP/s" if tensor else "GB/s",
                        "frac": round(ach / peak, 4),
                        "share_of_step": round(prof_ms[i] / timed_steps / (ms / args.steps), 4)}
    dom = max(per_class, key=lambda c: per_class[c]["share_of_step"]) if per_class else None
    roof = None
    if dom:
        e = per_class[dom]
        tensor = e["bound"] == "tensor"
        roof = {"kernel": e["kernel"], "bound": e["bound"], "achieved": e["achieved"],
                "peak": pk["bf16_tflops_sustained"] if tensor else pk["hbm_gbs"],
                "unit": e["unit"], "frac": e["frac"],
                "traffic": stored_traffic(e["kernel"], w.name),
                "algorithmic_per_launch": e["flops_per_launch"] if tensor else e["bytes_per_launch"],
                "peak_kind": pk_kind + (" bf16_tflops_sustained (kernel timed inside a long step)"
                                        if tensor else " hbm_gbs (copy)"),
                "timing": ("CUDA events inside the timed replays" if inline_events else
                           "CUDA events in separate replays of the same steps")}
    step_bytes = sum(ab[k] for k in ("embed", "lm_head", "dit_gemm", "attn", "context", "verify"))
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "blocks/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded fm_synth inputs; no trained weights)",
        "config": workload_config(w, R, world),
        "verified_tokens_per_s": round(tok_per_s, 1),
        "mean_accepted": round(n_sum / (args.steps * B), 3),
        "acceptance": acc,
        "step_hbm_gbs": round(step_bytes / (ms / args.steps / 1e3) / 1e9, 1),
        "step_hbm_frac": round(step_bytes / (ms / args.steps / 1e3) / 1e9 / pk["hbm_gbs"], 4),
        "roofline": roof, "kernels": per_class,
        "eager_profile_us_per_step": {k: v["us_per_step"] for k, v in eager.items()},
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "cuda_graphs": bool(graphs),
        "clocks": clk.summary(), "setup_s": round(setup_s, 1),
    }

    # end to end: host inputs in pinned memory, copies inside the timed region
    log(f"device-resident: {ms / args.steps:.4f} ms/step")
    if not args.no_e2e:
        RE = min(R, 8)
        pin = []
        for i in range(RE):
            rd = rounds[i]
            pin.append({k: (v.cpu().pin_memory() if v is not None else None) for k, v in rd.items()})
        # two device input buffers: a copy stream uploads step k+1's inputs
        # while step k runs (events order each upload after the step that
        # last read its buffer, and each step after its upload)
        dev_in = [{k: (torch.empty_like(v) if v is not None else None) for k, v in rounds[0].items()}
                  for _ in range(2)]
        # two sets of device outputs, one per input buffer: the copy stream
        # reads step k's results (accepted lengths and tokens) back while
        # step k + 1 writes the other set
        n_stage = [torch.zeros(B, dtype=torch.int32, device="cuda") for _ in range(2)]
        outs = [(torch.empty(B, dtype=torch.int32, device="cuda"),
                 torch.empty((B, K + 1), dtype=torch.int32, device="cuda")) for _ in range(2)]
        host_n = torch.empty((args.steps, B), dtype=torch.int32).pin_memory()
        host_tok = torch.empty((args.steps, B, K + 1), dtype=torch.int32).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in pin[0].values() if v is not None)
        d2h = B * 4 + B * (K + 1) * 4
        gstage = [None, None]
        if graphs:
            for bi in range(2):
                for key, v in pin[0].items():
                    if v is not None:
                        dev_in[bi][key].copy_(v)
                gstage[bi] = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gstage[bi]):
                    step(dev_in[bi], n_stage[bi], torch.cuda.current_stream(), outs[bi])
        torch.cuda.synchronize()
        barrier()
        cs = torch.cuda.Stream()
        copied = [torch.cuda.Event(), torch.cuda.Event()]
        used = [torch.cuda.Event(), torch.cuda.Event()]
        read = [torch.cuda.Event(), torch.cuda.Event()]

        def upload(k: int, bi: int):
            with torch.cuda.stream(cs):
                if k >= 2:
                    cs.wait_event(used[bi])
                for key, v in pin[k % RE].items():
                    if v is not None:
                        dev_in[bi][key].copy_(v, non_blocking=True)
                copied[bi].record(cs)

        def download(k: int, bi: int):
            with torch.cuda.stream(cs):
                cs.wait_event(used[bi])
                host_n[k].copy_(n_stage[bi], non_blocking=True)
                host_tok[k].copy_(outs[bi][1], non_blocking=True)
                read[bi].record(cs)

        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cs.wait_event(e0)
        upload(0, 0)
        for k in range(args.steps):
            bi = k % 2
            if k + 1 < args.steps:
                upload(k + 1, 1 - bi)
            stream.wait_event(copied[bi])
            if k >= 2:
                stream.wait_event(read[bi])     # step k - 2's results are read
            if gstage[bi] is not None:
                gstage[bi].replay()
            else:
                step(dev_in[bi], n_stage[bi], stream, outs[bi])
            used[bi].record(stream)
            download(k, bi)
        stream.wait_stream(cs)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1))
        line["e2e"] = {"value": round(B * N * args.steps * world / (ems / 1e3), 3),
                       "unit": "blocks/s", "h2d_bytes_per_step": int(h2d),
                       "d2h_bytes_per_step": int(d2h), "ms_per_step": round(ems / args.steps, 5)}
    if factorised:
        # ablation, untimed: the same rounds drafted factorised (position i
        # from its own independent noise block), verified against the same
        # synthetic targets; those targets are built around the joint draft
        # of a random-weight drafter, so this compares the two paths on one
        # footing, not the trained drafters of the pages
        n_f = torch.zeros((R, B), dtype=torch.int32, device="cuda")
        for i in range(R):
            rd = rounds[i]
            if w.new_rows:
                fmb.fm_project_context(ctx.ctx, seqs, rd["hidden"], w.new_rows, [w.ctx] * B, stream)
            Xf = to_device(fs.factorised_noise(w, round_seed(i, rank)), w.dtype)
            tok_f, _ = ctx.draft_factorised(seqs, Xf, w.t_grid, w.temps, logits=False)
            fmb.fm_verify_greedy(ctx.ctx, rd["target"], tok_f.view(B, 1, K).contiguous(), B, 1, K, V,
                                 n_f[i], branch, out_tok, stream)
            del Xf
        torch.cuda.synchronize()
        line["ablation"] = {
            "joint": acceptance_stats(n_all, K),
            "factorised": acceptance_stats(n_f.cpu().numpy(), K),
            "rounds": R,
            "targets": "the joint draft's synthetic targets (random-weight drafter)"}
    ctx.close()
    if dist is not None:
        dist.destroy_process_group()
    return line


# ---------------------------------------------------------------- oracle (CPU) arm
def oracle_rounds(w: fs.Workload, budget_s: float, max_rounds: int, warmup: int = 0):
    """Time the fp64 oracle doing whole rounds of sequence 0 (context rows,
    draft, verify); returns (seconds per block, rounds timed, cores)."""
    from oracle import flashmap as om
    s = w.shape
    W = {k: v.astype(np.float64) for k, v in fs.make_weights(s, w.dtype).items()}
    base = fs.prefill_hidden(w, 0)
    C0, kv0 = om.project_context(W, s.n_blocks, base)
    times = []
    for r in range(warmup + max_rounds):
        ri = fs.round_inputs(dataclasses_replace_B1(w), r)
        t0 = time.perf_counter()
        if w.new_rows:
            _, kvn = om.project_context(W, s.n_blocks, ri.new_hidden[0])
            kv = [(np.concatenate([a, an]), np.concatenate([b, bn]))
                  for (a, b), (an, bn) in zip(kv0, kvn)]
        else:
            kv = kv0
        res = om.draft(W, s, kv, ri.noise[0], w.t_grid, w.temps[0], ri.u_draft[0])
        t1 = time.perf_counter()
        tgt = fs.target_logits(dataclasses_replace_B1(w), r, res["tokens"][None],
                               res["logits"][None].astype(np.float32))
        t2 = time.perf_counter()
        if w.temps[0] == 0:
            om.verify_greedy(tgt[0], res["tokens"])
        else:
            om.verify_sample(tgt[0], res["logits"].astype(np.float32), res["tokens"], w.temps[0],
                             ri.u_accept[0], ri.u_res[0])
        t3 = time.perf_counter()
        if r >= warmup:
            times.append((t1 - t0) + (t3 - t2))
        if r >= warmup and sum(times) > budget_s:
            break
    cores = len(os.sched_getaffinity(0))
    return times, cores


def dataclasses_replace_B1(w):
    import dataclasses
    return dataclasses.replace(w, B=1, temps=w.temps[:1])


def run_reference(args, w, world: int = 1):
    wr = dataclasses_replace_B1(w)
    times, cores = oracle_rounds(w, budget_s=1e9, max_rounds=args.steps, warmup=args.warmup)
    sec = sum(times)
    blocks = len(times) * wr.n_noise
    v = blocks / sec
    sample = (f"{len(times)} whole rounds of sequence 0 of {w.name} (context rows, "
              f"{wr.n_noise} noise draft(s) x K={w.shape.K}, verify) per timed step set")
    return {"impl": "reference", "metric": METRIC, "value": round(v, 5), "unit": "blocks/s",
            "n_gpus": world, "steps": len(times), "warmup": args.warmup,
            "ms_per_step": round(sec / len(times) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded fm_synth inputs; no trained weights)",
            "config": workload_config(w, len(times) + args.warmup, world),
            "cpu_baseline": {"value": round(v, 5), "unit": "blocks/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(v, 5), "unit": "blocks/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def log(msg):
    print(f"[bench] {msg}", file=sys.stderr, flush=True)


# ---------------------------------------------------------------- local ranks
def _rank_entry(env: dict, entry, entry_args) -> None:
    os.environ.update(env)
    rc = entry(*entry_args)
    sys.exit(int(rc or 0))


def launch_local(n: int, entry, *entry_args, timeout_s: float = 3600.0) -> None:
    """Start n local ranks, one process each, with the environment a torchrun
    launch gives them (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_ADDR=127.0.0.1,
    MASTER_PORT), run entry(*entry_args) in each, and wait.  Raises when a
    rank fails or outlives the timeout (it is then terminated)."""
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    ctx = mp.get_context("spawn")
    procs = []
    for r in range(n):
        env = {"RANK": str(r), "LOCAL_RANK": str(r), "WORLD_SIZE": str(n),
               "LOCAL_WORLD_SIZE": str(n), "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)}
        p = ctx.Process(target=_rank_entry, args=(env, entry, entry_args))
        p.start()
        procs.append(p)
    t_end = time.time() + timeout_s
    codes = []
    for p in procs:
        p.join(max(1.0, t_end - time.time()))
        if p.is_alive():
            p.terminate()
            p.join(30)
        codes.append(p.exitcode)
    if any(c != 0 for c in codes):
        raise RuntimeError(f"local ranks exited with codes {codes}")


def main():
    faulthandler.enable()
    args = parse()
    launched = "WORLD_SIZE" in os.environ
    if args.impl == "fm" and args.gpus > 1 and not launched:
        # no launcher: start one rank per GPU here (replicas, NCCL for the
        # barrier and the two reductions), each re-running this entry point
        launch_local(args.gpus, main)
        return 0
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus if args.impl == "reference" else 1)))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = fs.WORKLOADS[args.workload]
    if args.impl == "reference":
        if rank != 0:
            return 0
        # rank 0 alone times the oracle on the host cores for the job
        print(json.dumps(run_reference(args, w, world)), flush=True)
        return 0
    line = run_fm(args, w, rank, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            log("timing the oracle on host cores")
            times, cores = oracle_rounds(w, budget_s=args.cpu_seconds, max_rounds=64, warmup=0)
            line["cpu_baseline"] = {
                "value": round(len(times) * w.n_noise / sum(times), 5), "unit": "blocks/s",
                "cores": cores, "kind": "oracle",
                "sample": f"{len(times)} rounds of sequence 0 of {w.name}, fp64 numpy/BLAS, "
                          f"~{args.cpu_seconds:.0f} s budget"}
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
